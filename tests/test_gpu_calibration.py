"""GPU: the output-error kernel and the accumulated-error calibration.

lite_attn_output_error is checked against numpy fp64 sums.  The calibration
is checked for what defines it: replaying its schedule reproduces each step's
error (up to the order of the kernel's fp64 atomic sums) and stays within budget, each chosen threshold is the most
aggressive one of the grid that fits (the next one up breaks the budget from
the same carried mask), and the replayed steps match the oracle.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import liteattn, synthetic
from temporal_block_sparse_sm_b200.calibration import calibrate, error_budgets, threshold_grid
from tests.helpers import bf16_bits, bits_to_f64
from tests.parity import check_step, pick_items

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


@pytest.mark.parametrize("shape,layout", [((2, 3, 1000, 64), "bhnd"), ((1, 12, 8192, 128), "bhnd"),
                                          ((2, 3, 1000, 128), "bnhd")])
def test_output_error_matches_numpy(shape, layout):
    B, H, N, d = shape
    plan = liteattn.Plan(B, H, N, d, d, d, [-1.0], layout=layout)
    g = torch.Generator(device="cuda").manual_seed(5)
    ref = torch.randn(plan.shape, generator=g, device="cuda").to(torch.bfloat16)
    o = (ref.float() + 0.01 * torch.randn(plan.shape, generator=g, device="cuda")).to(torch.bfloat16)
    e = plan.output_error(o, ref)
    a, b = bits_to_f64(bf16_bits(o)), bits_to_f64(bf16_bits(ref))
    diff = np.abs(a - b)
    assert e["sum_abs_diff"] == pytest.approx(diff.sum(), rel=1e-6)
    assert e["sum_abs_ref"] == pytest.approx(np.abs(b).sum(), rel=1e-6)
    assert e["max_abs"] == diff.max()
    same = plan.output_error(ref, ref)
    assert same["sum_abs_diff"] == 0.0 and same["max_abs"] == 0.0 and same["rel_l1"] == 0.0


def _plans(cfg, taus):
    return liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, taus)


@pytest.mark.parametrize("cfg_name,total", [("c1", 1e-3), ("c2", 5e-3)])
def test_calibration_is_reproducible_tight_and_matches_oracle(cfg_name, total):
    cfg = synthetic.CONFIGS[cfg_name]
    T = cfg.T
    wl = synthetic.Workload(cfg, seed=0, device="cuda")
    inputs = [wl.inputs(t) for t in range(T)]
    grid = threshold_grid()
    grid_plan, dense_plan = _plans(cfg, grid), _plans(cfg, [-math.inf])
    budgets = error_budgets(T, total)
    new_o = lambda: torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
    res = calibrate(grid_plan, dense_plan, lambda t: inputs[t], budgets, new_o)
    print(cfg_name, "taus", [round(x, 2) for x in res.taus], "errors", [f"{e:.2e}" for e in res.errors],
          "over", res.over_budget, "trials", res.trials)
    assert len(res.taus) == T

    # replay the calibrated schedule in propagate mode on the same inputs
    plan = _plans(cfg, res.taus)
    mask, dmask = plan.mask(), dense_plan.mask()
    probe = grid_plan.mask()
    o, od = new_o(), new_o()
    for t in range(T):
        q, k, v = inputs[t]
        dmask.reset()
        dense_plan.step(q, k, v, od, dmask, dmask, 0)
        bits_in = mask.export_bits()
        plan.step(q, k, v, o, mask, mask, t)
        err = plan.output_error(o, od)["rel_l1"]
        # the kernel is deterministic; only the order of the fp64 atomic sums may vary
        assert err == pytest.approx(res.errors[t], rel=1e-9, abs=1e-15), f"step {t}: replay {err} vs {res.errors[t]}"
        if t not in res.over_budget:
            assert err <= budgets[t] * (1 + 1e-9)
        gi = grid.index(res.taus[t])
        if gi > 0:   # the next more aggressive threshold breaks the budget from the same mask
            probe.import_bits(bits_in)
            grid_plan.step(q, k, v, o, probe, probe, gi - 1)
            assert grid_plan.output_error(o, od)["rel_l1"] > budgets[t] * (1 - 1e-9)
            # recompute this step's own output (same mask, same threshold) for the parity check below
            probe.import_bits(bits_in)
            grid_plan.step(q, k, v, o, probe, probe, gi)
        bits_out = mask.export_bits()
        items = np.arange(plan.R) if cfg_name == "c1" else pick_items(cfg.B, cfg.H, plan.Tq, 32, 300 + t)
        check_step(q, k, v, o, bits_in, bits_out, B=cfg.B, H=cfg.H, N=cfg.N, d=cfg.d, Br=cfg.Br, Bc=cfg.Bc,
                   tau=res.taus[t], items=items, step=t)
