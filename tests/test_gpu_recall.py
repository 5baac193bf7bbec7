"""GPU parity of the fixed-recall skip predicate against its oracle.

The predicate ("Training-free sparse attention based on cumulative energy
filtering", abstract: a fixed recall rate held by a dynamic threshold inside
the FlashAttention pass) is the plan's per-step test instead of the QK-Skip
threshold; ``oracle.step_recall`` restates it and ``tests/parity.py`` compares
(masks within the decision margin, outputs within max-abs 1e-2 / mean-abs
1e-3).  Every test goes through the C ABI on seeded synthetic inputs.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from temporal_block_sparse_sm_b200 import liteattn, synthetic
from tests.parity import check_step, pick_items

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


def _run(cfg, ps, check_steps, n_items=None, mode="propagate", seed=0, layout="bhnd"):
    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, ps, predicate="recall", layout=layout)
    assert liteattn.lite_attn_plan_predicate(plan.handle) == liteattn.LITE_PRED_RECALL
    mask = plan.mask()
    wl = synthetic.Workload(cfg, seed=seed, device="cuda")
    o = torch.empty(plan.shape, dtype=torch.bfloat16, device="cuda")
    out = []
    for t in range(len(ps)):
        q, k, v = wl.inputs(t)
        if layout == "bnhd":
            q, k, v = (x.transpose(1, 2).contiguous() for x in (q, k, v))
        if mode == "recompute":
            mask.reset()
        check = t in check_steps
        if check:
            bits_in = mask.export_bits()
        plan.step(q, k, v, o, mask, mask, t)
        if check:
            bits_out = mask.export_bits()
            items = np.arange(plan.R) if n_items is None else pick_items(cfg.B, cfg.H, plan.Tq, n_items, 97 * t + seed)
            back = (lambda x: x.transpose(1, 2).contiguous()) if layout == "bnhd" else (lambda x: x)
            res = check_step(back(q), back(k), back(v), back(o), bits_in, bits_out, B=cfg.B, H=cfg.H, N=cfg.N,
                             d=cfg.d, Br=cfg.Br, Bc=cfg.Bc, p=plan.taus[t], items=items, step=t)
            st = plan.stats(mask)
            assert st["device_status"] == 0
            assert st["live_out"] == int(oracle.bits_to_bool(bits_out, plan.Tk).sum())
            out.append((res, st))
    torch.cuda.synchronize()
    return plan, mask, out


@pytest.mark.parametrize("mode", ["propagate", "recompute"])
@pytest.mark.parametrize("p", [0.9, 0.99])
def test_c1_every_item(p, mode):
    cfg = synthetic.CONFIGS["c1"]
    _, _, out = _run(cfg, [p] * cfg.T, check_steps=range(cfg.T), mode=mode)
    for r, st in out:
        print("c1", p, mode, r)
    assert out[-1][1]["skip_fraction"] > 0.0, "the predicate should skip tiles on the locality workload"


@pytest.mark.parametrize("mode", ["propagate", "recompute"])
@pytest.mark.parametrize("p", [0.9, 0.99, 0.999])
def test_c5_shape_several_recall_targets(p, mode):
    """The skip-sweep shape (N = 32760, H = 12, d = 128), 20 steps at one recall
    target; 64 sampled query tiles (first and partial last included) at steps 0,
    10 and 19."""
    cfg = synthetic.CONFIGS["c5"]
    _, _, out = _run(cfg, [p] * cfg.T, check_steps=(0, 10, cfg.T - 1), n_items=64, mode=mode)
    for r, st in out:
        print("c5 recall", p, mode, r, "skip", round(st["skip_fraction"], 4))
    assert out[-1][1]["skip_fraction"] > 0.0


def test_recall_one_is_dense_and_matches_the_threshold_kernel_at_minus_inf():
    """p = 1 skips nothing, so its outputs equal, bit for bit, those of a QK-Skip
    plan at tau = -inf on the same inputs (same tiles, same arithmetic)."""
    cfg = synthetic.CONFIGS["c2"]
    wl = synthetic.Workload(cfg, seed=2, device="cuda")
    q, k, v = wl.inputs(0)
    pr = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, [1.0], predicate="recall")
    pt = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, [-math.inf])
    mr, mt = pr.mask(), pt.mask()
    o1, o2 = torch.empty_like(q), torch.empty_like(q)
    pr.step(q, k, v, o1, mr, mr, 0)
    pt.step(q, k, v, o2, mt, mt, 0)
    torch.cuda.synchronize()
    assert pr.stats(mr)["live_out"] == pr.stats(mr)["tiles_total"]
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 65, 200, 1000])
def test_edge_shapes(d, N):
    Bsz, H = (2, 3) if d == 64 else (1, 2)
    cfg = synthetic.WorkloadConfig("edge", Bsz, H, N, d, d, d, (1, 1, N), 2, 0.05, 0.0)
    _run(cfg, [0.9, 0.5], check_steps=(0, 1), seed=3)


def test_token_major_layout():
    cfg = synthetic.CONFIGS["c2"]
    import dataclasses
    cfg = dataclasses.replace(cfg, T=3)
    _, _, out = _run(cfg, [0.95] * 3, check_steps=(0, 1, 2), n_items=48, layout="bnhd")
    for r, st in out:
        print("c2 bnhd recall", r)
