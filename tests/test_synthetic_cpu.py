"""The seeded input generator (CPU, no GPU).

Every workload the tests and the benchmark use comes from
temporal_block_sparse_sm_b200/synthetic.py.  These tests hold it to the
recipe in its header:
  * tokens in row-major (frame, y, x) order;
  * |phi|^2 = d/2, with pair p on axis p mod 3 at the stated angular rate;
  * q0 = 2 phi + 0.5 N(0,1) and k0 likewise, so the mean self logit
    q.k / sqrt(d) is 2 sqrt(d);
  * per-step noise of size sigma, seeded generators, and any step produced on
    its own;
  * imported masks: random ones at the requested live fraction, locality ones
    that keep each query tile's nearest key tiles, bits past Tk always 0;
  * the workloads' threshold schedules.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import synthetic


@pytest.mark.parametrize("grid", [(4, 16, 16), (3, 5, 7), (1, 1, 9)])
def test_positions_are_row_major_frame_y_x(grid):
    F, Y, X = grid
    pos = synthetic.positions(grid)
    assert pos.shape == (F * Y * X, 3)
    n = (pos[:, 0] * Y + pos[:, 1]) * X + pos[:, 2]
    assert torch.equal(n, torch.arange(F * Y * X))


@pytest.mark.parametrize("grid,d", [((4, 16, 16), 64), ((21, 30, 52), 128), ((2, 3, 5), 128)])
def test_phi_norm_axes_and_rates(grid, d):
    ph = synthetic.phi(grid, d)
    pos = synthetic.positions(grid).to(torch.float64)
    assert ph.shape == (pos.shape[0], d)
    assert torch.allclose((ph * ph).sum(1), torch.full((pos.shape[0],), d / 2, dtype=torch.float64), atol=1e-9)
    pairs = d // 2
    counts = [len(range(a, pairs, 3)) for a in range(3)]
    for p in (0, 1, 2, 3, pairs - 1):
        a, rank = p % 3, p // 3
        L = float(grid[a])
        w = L ** (-rank / counts[a]) if L > 1 else 1.0
        assert torch.allclose(ph[:, 2 * p], torch.cos(w * pos[:, a]), atol=1e-12)
        assert torch.allclose(ph[:, 2 * p + 1], torch.sin(w * pos[:, a]), atol=1e-12)
    # rank 0 of every axis turns at 1 rad/token
    assert torch.allclose(ph[:, 0], torch.cos(pos[:, 0]), atol=1e-12)


def test_phi_rejects_odd_dimensions():
    with pytest.raises(ValueError):
        synthetic.phi((2, 2, 2), 63)


def _small_cfg(sigma=0.05, drift=0.0, d=64):
    return synthetic.WorkloadConfig("t", 2, 3, 256, d, d, d, (4, 8, 8), 4, sigma, drift)


def test_workload_is_seeded_and_steps_are_independent():
    cfg = _small_cfg(drift=0.01)
    a, b = synthetic.Workload(cfg, seed=3), synthetic.Workload(cfg, seed=3)
    c = synthetic.Workload(cfg, seed=4)
    for t in (0, 2):
        xa, xb, xc = a.inputs(t), b.inputs(t), c.inputs(t)
        for u, w, z in zip(xa, xb, xc):
            assert u.dtype == torch.bfloat16 and u.shape == (2, 3, 256, 64)
            assert torch.equal(u, w)
            assert not torch.equal(u, z)
    # step 2 does not depend on having produced steps 0 and 1 first
    fresh = synthetic.Workload(cfg, seed=3)
    assert all(torch.equal(u, w) for u, w in zip(fresh.inputs(2), a.inputs(2)))


def test_step_noise_and_self_logit_follow_the_recipe():
    d, sigma = 128, 0.05
    cfg = synthetic.WorkloadConfig("t", 1, 4, 2048, d, d, d, (2, 32, 32), 3, sigma, 0.0)
    wl = synthetic.Workload(cfg, seed=1)
    q0, k0, v0 = (x.double() for x in wl.inputs(0))
    q1 = wl.inputs(1)[0].double()
    # consecutive steps differ by sigma * (eps_1 - eps_0): std sigma * sqrt(2), plus bf16 rounding
    diff_std = float((q1 - q0).std())
    assert abs(diff_std - sigma * math.sqrt(2)) < 0.25 * sigma * math.sqrt(2), diff_std
    # v0 ~ N(0, 1)
    assert abs(float(v0.mean())) < 0.01 and abs(float(v0.std()) - 1.0) < 0.01
    # mean self logit q.k / sqrt(d) = 4 |phi|^2 / sqrt(d) = 2 sqrt(d)
    self_logit = (q0 * k0).sum(-1) / math.sqrt(d)
    assert abs(float(self_logit.mean()) - 2 * math.sqrt(d)) < 0.02 * 2 * math.sqrt(d), float(self_logit.mean())


@pytest.mark.parametrize("Tk", [5, 32, 70])
@pytest.mark.parametrize("frac", [0.2, 0.8])
def test_random_live_bits(Tk, frac):
    rows = 400
    bits = synthetic.random_live_bits(rows, Tk, frac, seed=9).numpy().astype(np.uint32)
    W = -(-Tk // 32)
    assert bits.shape == (rows, W)
    live = ((bits[:, np.arange(Tk) >> 5] >> (np.arange(Tk) & 31).astype(np.uint32)) & 1).astype(bool)
    assert live[:, 0].all()                                   # keep_first
    assert abs(live[:, 1:].mean() - frac) < 0.05
    if Tk % 32:
        assert not (bits[:, W - 1] >> np.uint32(Tk % 32)).any(), "bits past Tk must be 0"
    again = synthetic.random_live_bits(rows, Tk, frac, seed=9).numpy().astype(np.uint32)
    assert np.array_equal(bits, again)


@pytest.mark.parametrize("frac", [0.2, 0.5, 1.0])
def test_locality_live_bits_keep_the_nearest_tiles(frac):
    grid, Br, Bc, B, H = (4, 8, 8), 64, 64, 2, 3
    bits = synthetic.locality_live_bits(grid, B, H, Br, Bc, frac).numpy().astype(np.uint32)
    N = grid[0] * grid[1] * grid[2]
    Tq, Tk = -(-N // Br), -(-N // Bc)
    assert bits.shape == (B * H * Tq, -(-Tk // 32))
    live = ((bits[:, np.arange(Tk) >> 5] >> (np.arange(Tk) & 31).astype(np.uint32)) & 1).astype(bool)
    keep = math.ceil(frac * Tk)
    assert (live.sum(1) == keep).all()
    assert np.array_equal(live[:Tq], live[Tq:2 * Tq]), "every (batch, head) gets the same pattern"
    pos = synthetic.positions(grid).double()
    qc = torch.stack([pos[i * Br:(i + 1) * Br].mean(0) for i in range(Tq)])
    kc = torch.stack([pos[j * Bc:(j + 1) * Bc].mean(0) for j in range(Tk)])
    dist = torch.cdist(qc, kc).numpy()
    for i in range(Tq):
        assert live[i, i], "a query tile keeps its own diagonal key tile"
        kept, dropped = dist[i, live[i]], dist[i, ~live[i]]
        if dropped.size:
            assert kept.max() <= dropped.min() + 1e-9, "kept tiles are the nearest ones"


def test_schedules():
    c2 = synthetic.CONFIGS["c2"].taus()
    assert len(c2) == 10
    assert c2[0] == pytest.approx(math.log(1e-6)) and c2[-1] == pytest.approx(math.log(1e-3))
    assert all(b > a for a, b in zip(c2, c2[1:]))
    steps = np.diff(c2)
    assert np.allclose(steps, steps[0]), "linear in the log domain"
    assert synthetic.CONFIGS["c1"].taus() == [pytest.approx(math.log(1e-4))] * 3
    c5 = synthetic.CONFIGS["c5"]
    assert math.isinf(c5.fixed_taus[-1]) and c5.fixed_taus[-1] < 0
    for name, cfg in synthetic.CONFIGS.items():
        assert cfg.grid[0] * cfg.grid[1] * cfg.grid[2] == cfg.N, name
