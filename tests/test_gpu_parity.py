"""GPU parity: the sm_100a LiteAttention step against the CPU oracle.

Every test goes through the C ABI (ctypes binding) on seeded synthetic
inputs and compares element by element with the oracle (tests/parity.py
states the acceptance rule).
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest
import torch

import oracle
from temporal_block_sparse_sm_b200 import liteattn, synthetic
from tests.helpers import bf16_bits, bits_to_f64, sdpa_f64
from tests.parity import check_step, pick_items, pick_items_per_head

pytestmark = pytest.mark.gpu

FULL = os.environ.get("LITE_FULL_PARITY", "0") == "1"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


def bench_pair_stride(cfg) -> int:
    """The pairing bench.py times by default (query tiles one video frame apart)."""
    import bench
    return bench.pair_stride_of(bench.parse_args([]).pair_stride, cfg)


def _run(cfg, seed, check_steps, n_items=None, mode="propagate", taus=None, full_steps=(), per_head=False,
         pair_stride=1):
    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, taus or cfg.taus(), pair_stride=pair_stride)
    mask = plan.mask()
    wl = synthetic.Workload(cfg, seed=seed, device="cuda")
    o = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
    out = []
    for t in range(cfg.T):
        q, k, v = wl.inputs(t)
        if mode == "recompute":
            mask.reset()
        check = t in check_steps
        if check:
            bits_in = mask.export_bits()
        plan.step(q, k, v, o, mask, mask, t)
        if check:
            bits_out = mask.export_bits()
            if n_items is None or t in full_steps:
                items = np.arange(plan.R)
            else:
                pick = pick_items_per_head if per_head else pick_items
                items = pick(cfg.B, cfg.H, plan.Tq, n_items, seed * 1000 + t)
            res = check_step(q, k, v, o, bits_in, bits_out, B=cfg.B, H=cfg.H, N=cfg.N, d=cfg.d, Br=cfg.Br,
                             Bc=cfg.Bc, tau=plan.taus[t], items=items, step=t)
            st = plan.stats(mask)
            assert st["device_status"] == 0
            assert st["live_out"] == int(oracle.bits_to_bool(bits_out, plan.Tk).sum())
            assert st["live_in"] == int(oracle.bits_to_bool(bits_in, plan.Tk).sum())
            out.append((res, st))
    torch.cuda.synchronize()
    return plan, mask, out


def test_c1_every_step_every_item():
    cfg = synthetic.CONFIGS["c1"]
    _, _, out = _run(cfg, 0, check_steps=range(cfg.T))
    assert len(out) == cfg.T
    for res, st in out:
        print(res)


@pytest.mark.parametrize("seed", [1, 2])
def test_c1_other_seeds(seed):
    cfg = synthetic.CONFIGS["c1"]
    _run(cfg, seed, check_steps=range(cfg.T))


def test_c1_recompute_mode():
    cfg = synthetic.CONFIGS["c1"]
    _, _, out = _run(cfg, 0, check_steps=range(cfg.T), mode="recompute")
    for res, st in out:
        assert st["live_in"] == st["tiles_total"]


def test_c2_trajectory():
    cfg = synthetic.CONFIGS["c2"]
    steps = range(cfg.T)
    _, _, out = _run(cfg, 0, check_steps=steps, n_items=None if FULL else 48, full_steps=(0, cfg.T - 1))
    skip = [r.skip_fraction for r, _ in out]
    print("c2 skip by step", skip)
    assert out[-1][1]["live_out"] <= out[0][1]["live_out"]
    assert out[-1][1]["skip_fraction"] > 0.05, "the schedule should kill tiles on this workload"


def test_c3_full_size_sampled():
    """Config 3 (N = 32760, H = 12, 50 steps): 64 sampled query tiles checked at
    every step of the full schedule, including the first and the partial last
    query tile; work items paired as bench.py pairs them."""
    cfg = synthetic.CONFIGS["c3"]
    _, _, out = _run(cfg, 0, check_steps=range(cfg.T), n_items=64, pair_stride=bench_pair_stride(cfg))
    assert len(out) == cfg.T
    for r, st in out:
        print("c3", r)


def test_c4_full_size_sampled():
    """Config 4 (N = 108000, H = 24, 50 steps): 32 sampled query tiles per head at
    steps 0, 10, 25 and 49 of the full schedule (the last two at the loosest
    thresholds, where most tiles die), in the launch configuration bench.py times
    (work items paired one video frame apart)."""
    cfg = synthetic.CONFIGS["c4"]
    checks = (0, 10, 25, 49)
    _, _, out = _run(cfg, 0, check_steps=checks, n_items=32, per_head=True, pair_stride=bench_pair_stride(cfg))
    assert all(r.n_items == 32 * cfg.H for r, _ in out)
    assert [r.step for r, _ in out] == list(checks)
    for r, st in out:
        print("c4", r)


C5_TAUS = synthetic.CONFIGS["c5"].fixed_taus


@pytest.mark.parametrize("mode", ["propagate", "recompute"])
@pytest.mark.parametrize("tau", C5_TAUS, ids=[("-inf" if math.isinf(t) else f"ln{math.exp(t):.0e}") for t in C5_TAUS])
def test_c5_fixed_threshold_sweep(tau, mode):
    """Config 5: 20 steps at one fixed threshold, in both modes; 64 sampled items
    (including the first and the partial last query tile) at steps 0, 10 and 19.
    tau = -inf must give dense attention: nothing skipped, and the oracle at
    -inf is pinned to library attention."""
    cfg = synthetic.CONFIGS["c5"]
    taus = [tau] * cfg.T
    _, _, out = _run(cfg, 0, check_steps=(0, 10, cfg.T - 1), n_items=64, mode=mode, taus=taus)
    for r, st in out:
        print("c5", mode, r)
    if math.isinf(tau):
        assert all(st["live_out"] == st["tiles_total"] for _, st in out)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 65, 127, 129, 200, 300, 1000])
def test_edge_shapes_against_oracle_and_dense(d, N):
    Bsz, H = (2, 3) if d == 64 else (1, 2)
    grid = (1, 1, N)
    cfg = synthetic.WorkloadConfig("edge", Bsz, H, N, d, d, d, grid, 2, 0.05, 0.0)
    taus = [-math.inf, math.log(1e-2)]
    plan, mask, out = _run(cfg, 3, check_steps=(0, 1), taus=taus)
    # step 0 at tau = -inf is dense attention: compare with the library routine too
    assert out[0][1]["newly_dead"] == 0


@pytest.mark.parametrize("d,grid", [(64, (2, 32, 32)), (128, (4, 32, 32))])
def test_tau_zero_keeps_only_rising_tiles(d, grid):
    """tau = 0 is the most aggressive threshold a plan accepts: a tile stays live
    only where some row's max reaches its running max (a tie stays live).  Three
    propagating steps on locality inputs, every work item against the oracle."""
    N = grid[0] * grid[1] * grid[2]
    cfg = synthetic.WorkloadConfig("tau0", 1, 2, N, d, d, d, grid, 3, 0.05, 0.0, schedule=("const", 0.0, 0.0))
    plan, mask, out = _run(cfg, 4, check_steps=(0, 1, 2))
    assert plan.taus == [0.0] * 3
    assert out[-1][1]["skip_fraction"] > 0.3, "tau = 0 should skip much of a locality workload"


def test_minus_inf_equals_library_dense_attention():
    B, H, N, d = 1, 2, 700, 128
    g = torch.Generator(device="cuda").manual_seed(7)
    q = torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16)
    o = torch.empty_like(q)
    plan = liteattn.Plan(B, H, N, d, d, d, [-math.inf])
    mask = plan.mask()
    plan.step(q, k, v, o, mask, mask, 0)
    torch.cuda.synchronize()
    ref = sdpa_f64(bits_to_f64(bf16_bits(q)), bits_to_f64(bf16_bits(k)), bits_to_f64(bf16_bits(v)))
    err = np.abs(o.double().cpu().numpy() - ref)
    assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())
    st = plan.stats(mask)
    assert st["newly_dead"] == 0 and st["live_out"] == st["tiles_total"]


@pytest.mark.parametrize("d", [64, 128])
def test_error_model_on_concentrated_attention(d):
    """Random q, k at twice unit scale make attention nearly one-hot, so outputs reach
    |o| in [2, 4) and beyond, where half a bf16 unit is 2^-7 and 2^-6: no bf16 output
    can meet an absolute 1e-2 there.  The arithmetic's own bound holds instead, per
    element: half a unit of the stored output, plus 2^-8 times the range of the values
    (P enters P.V as bf16, 2^-9 relative per weight, and the row sum uses the same
    rounded weights, so the output is a convex mix of the values with weights off by at
    most 2^-8 relative), plus fp32 slack."""
    B, H, N = 1, 2, 1500
    g = torch.Generator(device="cuda").manual_seed(21 + d)
    q, k = ((2.0 * torch.randn(B, H, N, d, generator=g, device="cuda")).to(torch.bfloat16) for _ in range(2))
    v = torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16)
    plan = liteattn.Plan(B, H, N, d, d, d, [-math.inf])
    mask = plan.mask()
    o = torch.empty_like(q)
    plan.step(q, k, v, o, mask, mask, 0)
    torch.cuda.synchronize()
    vf = bits_to_f64(bf16_bits(v))
    ref = sdpa_f64(bits_to_f64(bf16_bits(q)), bits_to_f64(bf16_bits(k)), vf)
    got = o.double().cpu().numpy()
    mag = np.maximum(np.abs(ref), np.abs(got))
    half_unit = np.where(mag > 0, 2.0 ** (np.floor(np.log2(np.maximum(mag, 1e-30))) - 8), 0.0)
    vrange = vf.max(axis=2, keepdims=True) - vf.min(axis=2, keepdims=True)
    bound = half_unit + 2.0 ** -8 * vrange + 1e-4
    err = np.abs(got - ref)
    assert (err <= bound).all(), float((err - bound).max())
    assert np.abs(ref).max() > 2.0, "the inputs must reach the large-|o| band"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("frac", [0.05, 0.3, 0.8])
def test_random_imported_masks(d, frac):
    N = 4000 if d == 128 else 2000
    cfg = synthetic.WorkloadConfig("imp", 1, 4, N, d, d, d, (1, 40, N // 40), 1, 0.05, 0.0)
    for tau in (-math.inf, math.log(1e-2)):
        plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, d, d, d, [tau])
        m_in, m_out = plan.mask(), plan.mask()
        bits = synthetic.random_live_bits(plan.R, plan.Tk, frac, seed=int(frac * 100) + d, keep_first=False)
        bits = bits.numpy().astype(np.uint32)
        m_in.import_bits(bits)
        wl = synthetic.Workload(cfg, seed=5, device="cuda")
        q, k, v = wl.inputs(0)
        o = torch.empty_like(q)
        plan.step(q, k, v, o, m_in, m_out, 0)
        bits_out = m_out.export_bits()
        assert np.array_equal(m_in.export_bits(), bits), "mask_in must not change when mask_out is separate"
        check_step(q, k, v, o, bits, bits_out, B=cfg.B, H=cfg.H, N=N, d=d, Br=d, Bc=d, tau=tau,
                   items=np.arange(plan.R))


def test_empty_mask_gives_zero_output():
    B, H, N, d = 1, 2, 600, 128
    plan = liteattn.Plan(B, H, N, d, d, d, [-1.0])
    m = plan.mask()
    m.import_bits(np.zeros((plan.R, plan.W), np.uint32))
    q = torch.randn(B, H, N, d, device="cuda").to(torch.bfloat16)
    o = torch.full_like(q, float("nan"))
    plan.step(q, q.clone(), q.clone(), o, m, m, 0)
    torch.cuda.synchronize()
    assert torch.all(o == 0)
    st = plan.stats(m)
    assert st["live_out"] == 0 and st["live_in"] == 0 and st["pv_tiles"] == 0


def test_in_place_and_separate_masks_agree_and_are_deterministic():
    cfg = synthetic.CONFIGS["c1"]
    wl = synthetic.Workload(cfg, seed=0, device="cuda")
    results = []
    for mode in ("inplace", "separate", "inplace"):
        plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, cfg.taus())
        a, b = plan.mask(), plan.mask()
        o = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
        outs = []
        for t in range(cfg.T):
            q, k, v = wl.inputs(t)
            if mode == "inplace":
                plan.step(q, k, v, o, a, a, t)
                cur = a
            else:
                src, dst = (a, b) if t % 2 == 0 else (b, a)
                plan.step(q, k, v, o, src, dst, t)
                cur = dst
            outs.append((o.clone(), cur.export_bits()))
        results.append(outs)
    for t in range(cfg.T):
        for other in results[1:]:
            assert torch.equal(results[0][t][0], other[t][0])
            assert np.array_equal(results[0][t][1], other[t][1])


def test_checkpoint_resume_matches_uninterrupted_run():
    cfg = synthetic.CONFIGS["c2"]
    wl = synthetic.Workload(cfg, seed=1, device="cuda")
    o1 = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, cfg.taus())
    m = plan.mask()
    for t in range(cfg.T):
        q, k, v = wl.inputs(t)
        plan.step(q, k, v, o1, m, m, t)
    full_bits = m.export_bits()
    # interrupted: 5 steps, checkpoint the mask, resume in a fresh plan
    plan_a = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, cfg.taus())
    ma = plan_a.mask()
    o2 = torch.empty_like(o1)
    for t in range(5):
        q, k, v = wl.inputs(t)
        plan_a.step(q, k, v, o2, ma, ma, t)
    ckpt = ma.export_bits()
    plan_b = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, cfg.taus())
    mb = plan_b.mask()
    mb.import_bits(ckpt)
    for t in range(5, cfg.T):
        q, k, v = wl.inputs(t)
        plan_b.step(q, k, v, o2, mb, mb, t)
    torch.cuda.synchronize()
    assert np.array_equal(mb.export_bits(), full_bits)
    assert torch.equal(o1, o2)


def test_outputs_fully_overwritten():
    cfg = synthetic.CONFIGS["c1"]
    wl = synthetic.Workload(cfg, seed=0, device="cuda")
    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, cfg.taus())
    m_in, m_out = plan.mask(), plan.mask()
    garbage = np.full((plan.R, plan.W), 0xA5A5A5A5 & ((1 << plan.Tk) - 1 if plan.Tk < 32 else 0xFFFFFFFF),
                      dtype=np.uint32)
    m_out.import_bits(garbage)
    q, k, v = wl.inputs(0)
    o = torch.full_like(q, float("nan"))
    plan.step(q, k, v, o, m_in, m_out, 0)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    bits = m_out.export_bits()
    ref = plan.mask()
    o2 = torch.empty_like(o)
    plan.step(q, k, v, o2, ref, ref, 0)
    assert np.array_equal(bits, ref.export_bits())
    assert torch.equal(o, o2)
