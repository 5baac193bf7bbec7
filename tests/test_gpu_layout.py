"""GPU: plans whose tensors are [B][N][H][d] (lite_attn_plan_create_ex).

The layout only moves rows in memory; the kernel's tiles, arithmetic and
decisions are the same.  So a [B][N][H][d] plan must give outputs and masks
bit-identical to a [B][H][N][d] plan on the same values, step after step,
and must match the oracle on its own.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import liteattn, synthetic
from tests.helpers import random_qkv
from tests.parity import check_step, pick_items

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


def _to_bnhd(x: torch.Tensor) -> torch.Tensor:
    return x.transpose(1, 2).contiguous()


def _run_both(B, H, N, d, taus, inputs):
    """Run the same steps on a [B,H,N,d] plan and a [B,N,H,d] plan; compare bit for bit."""
    p1 = liteattn.Plan(B, H, N, d, d, d, taus)
    p2 = liteattn.Plan(B, H, N, d, d, d, taus, layout="bnhd")
    assert p2.shape == (B, N, H, d)
    m1, m2 = p1.mask(), p2.mask()
    for t in range(len(taus)):
        q, k, v = inputs(t)
        qn, kn, vn = _to_bnhd(q), _to_bnhd(k), _to_bnhd(v)
        o1 = torch.full_like(q, float("nan"))
        o2 = torch.full_like(qn, float("nan"))
        p1.step(q, k, v, o1, m1, m1, t)
        p2.step(qn, kn, vn, o2, m2, m2, t)
        torch.cuda.synchronize()
        back = o2.transpose(1, 2).contiguous()
        assert torch.equal(back.view(torch.int16), o1.view(torch.int16)), f"step {t}: outputs differ"
        assert np.array_equal(m1.export_bits(), m2.export_bits()), f"step {t}: masks differ"
        s1, s2 = p1.stats(m1), p2.stats(m2)
        assert s1["live_out"] == s2["live_out"] and s1["newly_dead"] == s2["newly_dead"]
        assert s2["device_status"] == 0
    return p1.stats(m1)


@pytest.mark.parametrize("cfg_name", ["c1", "c2"])
def test_bnhd_equals_bhnd_on_workloads(cfg_name):
    cfg = synthetic.CONFIGS[cfg_name]
    T = min(cfg.T, 4)
    wl = synthetic.Workload(cfg, seed=0, device="cuda")
    st = _run_both(cfg.B, cfg.H, cfg.N, cfg.d, cfg.taus()[:T], wl.inputs)
    print(cfg_name, "skip after", T, "steps:", st["skip_fraction"])


@pytest.mark.parametrize("B,H,N,d", [(2, 3, 1000, 64), (2, 3, 1000, 128), (1, 5, 300, 128), (3, 1, 65, 64)])
def test_bnhd_equals_bhnd_on_edge_shapes(B, H, N, d):
    taus = [math.log(1e-2)] * 3
    dev = [tuple(torch.from_numpy(x).view(torch.bfloat16).cuda() for x in random_qkv(B, H, N, d, seed=40 + t,
                                                                                       scale_qk=2.0))
           for t in range(3)]
    st = _run_both(B, H, N, d, taus, lambda t: dev[t])
    assert st["newly_dead"] >= 0


@pytest.mark.parametrize("cfg_name", ["c1", "c2"])
def test_bnhd_matches_oracle(cfg_name):
    """[B][N][H][d] plans against the oracle on their own: every item of c1's 3
    steps; 64 sampled items (first and last query tiles included) at each of
    c2's 10 steps."""
    cfg = synthetic.CONFIGS[cfg_name]
    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, cfg.taus(), layout="bnhd")
    mask = plan.mask()
    wl = synthetic.Workload(cfg, seed=1, device="cuda")
    for t in range(cfg.T):
        q, k, v = wl.inputs(t)
        o = torch.full((cfg.B, cfg.N, cfg.H, cfg.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        bits_in = mask.export_bits()
        plan.step(_to_bnhd(q), _to_bnhd(k), _to_bnhd(v), o, mask, mask, t)
        bits_out = mask.export_bits()
        items = np.arange(plan.R) if cfg_name == "c1" else pick_items(cfg.B, cfg.H, plan.Tq, 64, 7 * t)
        res = check_step(q, k, v, o.transpose(1, 2).contiguous(), bits_in, bits_out, B=cfg.B, H=cfg.H, N=cfg.N,
                         d=cfg.d, Br=cfg.Br, Bc=cfg.Bc, tau=plan.taus[t], items=items, step=t)
        print(res)


def test_bnhd_rejects_bhnd_shaped_tensors():
    plan = liteattn.Plan(1, 2, 100, 64, 64, 64, [-1.0], layout="bnhd")
    mask = plan.mask()
    x = torch.zeros(1, 2, 100, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        plan.step(x, x, x, torch.empty_like(x), mask, mask, 0)
