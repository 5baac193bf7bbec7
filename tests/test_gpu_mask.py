"""GPU tests of the skip-mask store: reset, import/export round trips, and the
bitmask -> live-list compaction checked bit-exactly against numpy."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from temporal_block_sparse_sm_b200 import liteattn, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


def expected_lists(bits: np.ndarray, B: int, H: int, Tq: int, Tk: int, stride: int = 1):
    """Per query-tile pair (tests/pairing.py): ascending (j, flags) of the union of the two rows."""
    from tests.pairing import pairs
    live = oracle.bits_to_bool(bits, Tk).reshape(B * H, Tq, Tk)
    lists, cnts = [], []
    for bh in range(B * H):
        for qa, qb in pairs(Tq, stride):
            a = live[bh, qa]
            b = live[bh, qb] if qb >= 0 else np.zeros(Tk, bool)
            js = np.flatnonzero(a | b)
            ent = js.astype(np.uint64) | ((a[js].astype(np.uint64) | (b[js].astype(np.uint64) << 1)) << 30)
            lists.append(ent.astype(np.uint32))
            cnts.append(len(js))
    return lists, np.array(cnts)


def check_lists(plan, mask, bits):
    lst, cnt, order = mask.export_lists()
    exp_lists, exp_cnt = expected_lists(bits, plan.B, plan.H, plan.Tq, plan.Tk, plan.pair_stride)
    assert np.array_equal(cnt, exp_cnt)
    for g in range(plan.G):
        assert np.array_equal(lst[g, : cnt[g]], exp_lists[g]), g
    assert np.array_equal(np.sort(order), np.arange(plan.G))
    keys = (cnt[order].astype(np.int64) * 1024) // (plan.Tk + 1)
    assert np.all(np.diff(keys) <= 0), "work order must be longest-first"


@pytest.mark.parametrize("shape", [(1, 2, 1024, 64), (2, 3, 200, 64), (1, 2, 8192, 128), (1, 1, 70000, 64),
                                   (1, 3, 32760, 128), (1, 1, 1, 128)])
def test_reset_state(shape):
    B, H, N, d = shape
    plan = liteattn.Plan(B, H, N, d, d, d, [-1.0])
    m = plan.mask()
    bits = m.export_bits()
    full = oracle.all_live_rows(plan.R, N, d)
    assert np.array_equal(bits, full)
    check_lists(plan, m, bits)
    st = plan.stats(m)
    assert st["live_out"] == plan.R * plan.Tk and st["last_step"] == -1
    # reset after an import restores the all-live state
    m.import_bits(np.zeros_like(bits))
    m.reset()
    assert np.array_equal(m.export_bits(), full)


@pytest.mark.parametrize("shape", [(1, 2, 1024, 64), (2, 3, 200, 64), (1, 2, 8192, 128), (1, 1, 70000, 64),
                                   (1, 3, 32760, 128)])
@pytest.mark.parametrize("frac", [0.0, 0.02, 0.5, 0.97])
def test_import_export_and_compaction(shape, frac):
    B, H, N, d = shape
    plan = liteattn.Plan(B, H, N, d, d, d, [-1.0])
    m = plan.mask()
    bits = synthetic.random_live_bits(plan.R, plan.Tk, frac, seed=17, keep_first=False).numpy().astype(np.uint32)
    m.import_bits(bits)
    assert np.array_equal(m.export_bits(), bits)
    check_lists(plan, m, bits)
    st = plan.stats(m)
    assert st["live_out"] == int(oracle.bits_to_bool(bits, plan.Tk).sum())


def test_import_rejects_bits_past_tk():
    plan = liteattn.Plan(1, 1, 1000, 64, 64, 64, [-1.0])   # Tk = 16
    m = plan.mask()
    bits = np.zeros((plan.R, plan.W), np.uint32)
    bits[3, 0] = 1 << 20
    with pytest.raises(liteattn.LiteAttnError) as ei:
        m.import_bits(bits)
    assert ei.value.code == liteattn.LITE_ERR_INVALID_ARG


def test_step_stats_and_cumulative_counters():
    cfg = synthetic.CONFIGS["c1"]
    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, [math.log(1e-2)] * 3)
    m = plan.mask()
    wl = synthetic.Workload(cfg, seed=0, device="cuda")
    o = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
    cum_qk = cum_pv = 0
    for t in range(3):
        prev = int(oracle.bits_to_bool(m.export_bits(), plan.Tk).sum())
        q, k, v = wl.inputs(t)
        plan.step(q, k, v, o, m, m, t)
        st = plan.stats(m)
        now = int(oracle.bits_to_bool(m.export_bits(), plan.Tk).sum())
        assert st["live_in"] == prev and st["live_out"] == now and st["newly_dead"] == prev - now
        assert st["qk_tiles"] == prev and st["pv_tiles"] == now and st["last_step"] == t
        assert st["executed_flops"] == 2.0 * 64 * 64 * 64 * (prev + now)
        cum_qk += prev
        cum_pv += now
        assert st["cum_qk_tiles"] == cum_qk and st["cum_pv_tiles"] == cum_pv and st["cum_steps"] == t + 1
        check_lists(plan, m, m.export_bits())
    assert cum_pv < cum_qk


@pytest.mark.parametrize("N,head_major", [(108000, True), (65536, True), (32760, False)])
def test_work_order_is_head_major_when_a_heads_kv_exceeds_a_quarter_of_l2(N, head_major):
    """One head's K and V above 32 MB (4*N*d bytes at d = 128): pairs run in index
    (head-by-head) order so each head's K/V stays in L2; below it: longest first."""
    B, H, d = 1, 2, 128
    plan = liteattn.Plan(B, H, N, d, d, d, [-1.0])
    m = plan.mask()
    bits = synthetic.random_live_bits(plan.R, plan.Tk, 0.5, seed=3).numpy().astype(np.uint32)
    m.import_bits(bits)
    lst, cnt, order = m.export_lists()
    assert np.array_equal(np.sort(order), np.arange(plan.G))
    if head_major:
        assert np.array_equal(order, np.arange(plan.G))
    else:
        keys = (cnt[order].astype(np.int64) * 1024) // (plan.Tk + 1)
        assert np.all(np.diff(keys) <= 0)
        assert not np.array_equal(order, np.arange(plan.G))
