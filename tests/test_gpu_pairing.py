"""GPU: plans whose work items pair query tiles a stride apart (pair_stride).

The pairing only decides which two query tiles share a CTA and its key/value
loads; each tile still walks its own live tiles in ascending order with its own
softmax state.  So a strided plan must reproduce the adjacent plan bit for bit
(outputs, masks, statistics), under both skip predicates and both layouts, and
its compacted lists must be the unions of its pairs' rows (numpy).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import liteattn, synthetic
from tests.pairing import pairs
from tests.parity import check_step, pick_items
from tests.test_gpu_mask import check_lists

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


@pytest.mark.parametrize("N,s", [(8192, 4), (32760, 12), (1000, 3), (129, 5), (128, 7)])
def test_pair_tiles_follow_the_rule(N, s):
    plan = liteattn.Plan(1, 2, N, 128, 128, 128, [-1.0], pair_stride=s)
    got = [liteattn.lite_attn_plan_pair_tiles(plan.handle, p) for p in range((plan.Tq + 1) // 2)]
    assert got == pairs(plan.Tq, s)
    with pytest.raises(liteattn.LiteAttnError):
        liteattn.lite_attn_plan_pair_tiles(plan.handle, (plan.Tq + 1) // 2)


def test_stride_needs_128_row_tiles():
    with pytest.raises(liteattn.LiteAttnError):
        liteattn.Plan(1, 2, 1024, 64, 64, 64, [-1.0], pair_stride=2)


@pytest.mark.parametrize("cfg_name,s", [("c2", 4), ("c3", 12)])
@pytest.mark.parametrize("predicate", ["threshold", "recall"])
@pytest.mark.parametrize("layout", ["bhnd", "bnhd"])
def test_strided_plan_reproduces_the_adjacent_plan(cfg_name, s, predicate, layout):
    cfg = synthetic.CONFIGS[cfg_name]
    T = 4
    sched = cfg.taus()[:T] if predicate == "threshold" else [0.99, 0.95, 0.9, 0.9]
    # a loose last threshold so that tiles die and the pairs' lists differ
    if predicate == "threshold":
        sched = sched[:-1] + [math.log(1e-2)]
    wl = synthetic.Workload(cfg, seed=4, device="cuda")
    mk = lambda st: liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, sched, layout=layout,
                                  predicate=predicate, pair_stride=st)
    pa, ps = mk(1), mk(s)
    ma, ms = pa.mask(), ps.mask()
    oa = torch.empty(pa.shape, dtype=torch.bfloat16, device="cuda")
    os_ = torch.full(ps.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        q, k, v = wl.inputs(t)
        if layout == "bnhd":
            q, k, v = (x.transpose(1, 2).contiguous() for x in (q, k, v))
        pa.step(q, k, v, oa, ma, ma, t)
        ps.step(q, k, v, os_, ms, ms, t)
        torch.cuda.synchronize()
        assert torch.equal(oa.view(torch.int16), os_.view(torch.int16)), f"step {t}: outputs differ"
        bits = ms.export_bits()
        assert np.array_equal(ma.export_bits(), bits), f"step {t}: masks differ"
        sa, ss = pa.stats(ma), ps.stats(ms)
        for key in ("live_in", "live_out", "newly_dead", "cum_qk_tiles", "cum_pv_tiles"):
            assert sa[key] == ss[key], key
        check_lists(ps, ms, bits)
    assert ss["skip_fraction"] > 0.0


def test_strided_plan_against_the_oracle():
    """The 1.3B-DiT shape with a one-frame stride (12 tiles), 3 propagating steps at a
    loose threshold; 64 sampled query tiles per step against the oracle."""
    cfg = synthetic.CONFIGS["c3"]
    taus = [math.log(1e-4), math.log(1e-3), math.log(1e-2)]
    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, taus, pair_stride=12)
    mask = plan.mask()
    wl = synthetic.Workload(cfg, seed=0, device="cuda")
    o = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
    for t in range(3):
        q, k, v = wl.inputs(t)
        bits_in = mask.export_bits()
        plan.step(q, k, v, o, mask, mask, t)
        r = check_step(q, k, v, o, bits_in, mask.export_bits(), B=cfg.B, H=cfg.H, N=cfg.N, d=cfg.d, Br=cfg.Br,
                       Bc=cfg.Bc, tau=plan.taus[t], items=pick_items(cfg.B, cfg.H, plan.Tq, 64, 31 + t), step=t)
        print("c3 stride 12", r)


@pytest.mark.parametrize("frac", [0.2, 0.6])
def test_imported_locality_masks_compact_per_pair(frac):
    cfg = synthetic.CONFIGS["c5"]
    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, [-math.inf], pair_stride=12)
    m = plan.mask()
    bits = synthetic.locality_live_bits(cfg.grid, cfg.B, cfg.H, cfg.Br, cfg.Bc, frac).numpy().astype(np.uint32)
    m.import_bits(bits)
    check_lists(plan, m, bits)
    # the one-frame pairing shares more of each pair's list than adjacent pairs do
    adj = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, [-math.inf])
    ma = adj.mask()
    ma.import_bits(bits)
    assert ms_entries(m) < ms_entries(ma)


def ms_entries(mask):
    return int(mask.export_lists()[1].sum())
