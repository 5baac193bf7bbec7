"""The GPU-vs-oracle comparator itself (CPU, no GPU).

``tests.parity.check_step`` decides every GPU parity test, so it is checked
here on the CPU.  The stand-in for a correct kernel is the oracle's own result
(mask bits, outputs rounded to bf16).  It must pass.  Copies of it with one
planted mistake each must fail: a mask bit flipped far from the threshold, a
tile revived after it was dead on entry, one output element off, a small bias
on every output, two rows swapped, a NaN.  A decision that sits within the
rounding margin of the threshold must be accepted, with the oracle re-run
under the stand-in's decision.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import bf16_bits
from tests.parity import MARGIN, check_step

B, H, N, d, Br, Bc = 1, 2, 300, 64, 64, 64          # 5 x 5 tiles, ragged last tile (44 rows / columns)
Tq, Tk, W = oracle.tiles(N, Br, Bc)
ITEMS = np.arange(B * H * Tq)


@pytest.fixture(scope="module")
def case():
    # key tiles at different scales, so that the weak ones fall below the running max and die
    g = torch.Generator().manual_seed(21)
    q = 2.0 * torch.randn(B, H, N, d, generator=g)
    k = 2.0 * torch.randn(B, H, N, d, generator=g)
    for j, s in enumerate([1.0, 0.3, 1.0, 0.2, 0.6]):
        k[:, :, j * Bc:(j + 1) * Bc] *= s
    v = torch.randn(B, H, N, d, generator=g)
    qh, kh, vh = (bf16_bits(x.to(torch.bfloat16)) for x in (q, k, v))
    rng = np.random.default_rng(4)
    live = rng.random((len(ITEMS), Tk)) < 0.8
    live[:, 0] = True
    bits_in = oracle.bool_to_bits(live)
    tau = -0.5
    res = oracle.step(qh, kh, vh, B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, tau=tau, items=ITEMS, mask_in=bits_in)
    tested = ~np.isnan(res["D"])
    killed = tested & ~oracle.bits_to_bool(res["mask_out"], Tk)
    assert killed.sum() >= 3, "the fixture must kill some tiles in this step"
    assert (~live).sum() >= 3, "the fixture must have tiles dead on entry"
    return dict(qh=qh, kh=kh, vh=vh, bits_in=bits_in, tau=tau, res=res)


def _as_tensor(o_rows: np.ndarray) -> torch.Tensor:
    """oracle rows [items, Br, d] -> bf16 [B, H, N, d] (what a correct kernel stores)."""
    full = torch.from_numpy(o_rows.reshape(B, H, Tq * Br, d)[:, :, :N].copy())
    return full.to(torch.bfloat16)


def _check(c, o, bits_out, tau=None):
    dummy = torch.empty(0)
    return check_step(dummy, dummy, dummy, o, c["bits_in"], bits_out, B=B, H=H, N=N, d=d, Br=Br, Bc=Bc,
                      tau=c["tau"] if tau is None else tau, items=ITEMS, host_qkv=(c["qh"], c["kh"], c["vh"]))


def test_a_correct_result_passes(case):
    r = _check(case, _as_tensor(case["res"]["o"]), case["res"]["mask_out"])
    # correctly rounded outputs: no error against the rounded oracle, at most half a
    # bf16 unit against the exact one (2^-7 below |o| = 4), 2^-8 relative above 1
    assert r.flips == 0 and r.max_abs_rounded == 0.0
    assert r.max_abs <= 2.0 ** -7 and r.max_scaled <= 2.0 ** -8
    assert sum(n for n, _, _ in r.by_band.values()) == B * H * N * d


def test_a_stray_bit_past_the_last_key_tile_fails(case):
    bits = case["res"]["mask_out"].copy()
    bits[3, (Tk + 2) >> 5] |= np.uint32(1 << ((Tk + 2) & 31))
    with pytest.raises(AssertionError, match="past Tk"):
        _check(case, _as_tensor(case["res"]["o"]), bits)


def test_a_mask_bit_flipped_far_from_the_threshold_fails(case):
    res = case["res"]
    margin = np.abs(res["D"] - case["tau"])
    cand = np.argwhere(~np.isnan(res["D"]) & (margin > 10 * MARGIN))
    n_, j = cand[len(cand) // 2]
    bits = res["mask_out"].copy()
    bits[n_, j >> 5] ^= np.uint32(1 << (j & 31))
    with pytest.raises(AssertionError, match="outside the margin"):
        _check(case, _as_tensor(res["o"]), bits)


def test_a_tile_revived_after_dead_on_entry_fails(case):
    res = case["res"]
    dead_in = np.argwhere(~oracle.bits_to_bool(case["bits_in"], Tk))
    n_, j = dead_in[0]
    bits = res["mask_out"].copy()
    bits[n_, j >> 5] |= np.uint32(1 << (j & 31))
    with pytest.raises(AssertionError):
        _check(case, _as_tensor(res["o"]), bits)


@pytest.mark.parametrize("mistake", ["one_element", "bias", "swapped_rows", "nan", "last_row_dropped"])
def test_a_wrong_output_fails(case, mistake):
    res = case["res"]
    o = _as_tensor(res["o"]).float()
    if mistake == "one_element":
        o[0, 1, 77, 5] += 0.03
    elif mistake == "bias":
        o += 3e-3
    elif mistake == "swapped_rows":
        o[0, 0, [10, 11]] = o[0, 0, [11, 10]]
    elif mistake == "nan":
        o[0, 0, 299, 0] = float("nan")
    elif mistake == "last_row_dropped":
        o[0, 1, N - 1] = 0.0
    with pytest.raises(AssertionError):
        _check(case, o.to(torch.bfloat16), res["mask_out"])


def test_a_flip_within_the_margin_is_accepted_and_reforced(case):
    """Move tau to just above a tested tile's D: the oracle now kills that tile,
    a kernel whose rounding kept it live must still pass (counted as one flip).
    With D < 0 no row of that tile rises above its running max, so keeping it
    live changes no later decision."""
    res = case["res"]
    D = res["D"]
    cand = np.argwhere(~np.isnan(D) & np.isfinite(D) & (D < -0.01))
    n_, j = cand[0]
    tau1 = float(D[n_, j]) + MARGIN / 4
    base = oracle.step(case["qh"], case["kh"], case["vh"], B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, tau=tau1,
                       items=ITEMS, mask_in=case["bits_in"])
    assert not oracle.bits_to_bool(base["mask_out"], Tk)[n_, j], "the oracle kills the tile at tau1"
    force = np.full((len(ITEMS), Tk), -1, dtype=np.int8)
    force[n_, j] = 1
    kept = oracle.step(case["qh"], case["kh"], case["vh"], B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, tau=tau1,
                       items=ITEMS, mask_in=case["bits_in"], force=force)
    r = _check(case, _as_tensor(kept["o"]), kept["mask_out"], tau=tau1)
    assert r.flips >= 1
    assert math.isfinite(r.max_abs) and r.max_abs <= 2.0 ** -7 and r.max_abs_rounded == 0.0


# ------------------------------------------------------------------ the fixed-recall predicate
@pytest.fixture(scope="module")
def recall_case(case):
    p = 0.9
    res = oracle.step_recall(case["qh"], case["kh"], case["vh"], B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, p=p,
                             items=ITEMS, mask_in=case["bits_in"])
    tested = ~np.isnan(res["E"])
    assert (tested & ~oracle.bits_to_bool(res["mask_out"], Tk)).sum() >= 2, "the fixture must skip tiles"
    return dict(case, p=p, res=res)


def _check_recall(c, o, bits_out):
    dummy = torch.empty(0)
    return check_step(dummy, dummy, dummy, o, c["bits_in"], bits_out, B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, p=c["p"],
                      items=ITEMS, host_qkv=(c["qh"], c["kh"], c["vh"]))


def test_recall_correct_result_passes(recall_case):
    r = _check_recall(recall_case, _as_tensor(recall_case["res"]["o"]), recall_case["res"]["mask_out"])
    assert r.flips == 0 and r.max_abs_rounded == 0.0


def test_recall_flip_far_from_the_boundary_fails(recall_case):
    res = recall_case["res"]
    E = res["E"]
    cand = np.argwhere(~np.isnan(E) & np.isfinite(E) & (np.abs(E) > 0.1))
    n_, j = cand[0]
    bits = res["mask_out"].copy()
    bits[n_, j >> 5] ^= np.uint32(1 << (j & 31))
    with pytest.raises(AssertionError, match="outside the margin"):
        _check_recall(recall_case, _as_tensor(res["o"]), bits)


def test_recall_flip_within_the_margin_is_reforced_with_its_consequences(recall_case, monkeypatch):
    """A stand-in kernel takes the other decision at the tested tile closest to the
    boundary (which the margin is widened to cover), and then follows the
    predicate from the state that decision leaves: later decisions of that row may
    differ from the unforced oracle's.  The harness must accept it: the first
    difference is near, and the oracle re-run from the forced decision agrees with
    everything after it."""
    import tests.parity as parity
    res = recall_case["res"]
    E = res["E"]
    fin = ~np.isnan(E) & np.isfinite(E)
    n_, j = np.argwhere(fin & (np.abs(E) == np.abs(E[fin]).min()))[0]
    force = np.full((len(ITEMS), Tk), -1, dtype=np.int8)
    force[n_, j] = 0 if oracle.bits_to_bool(res["mask_out"], Tk)[n_, j] else 1
    flipped = oracle.step_recall(recall_case["qh"], recall_case["kh"], recall_case["vh"], B=B, H=H, N=N, d=d,
                                 Br=Br, Bc=Bc, p=recall_case["p"], items=ITEMS, mask_in=recall_case["bits_in"],
                                 force=force)
    monkeypatch.setattr(parity, "MARGIN_RECALL", 2.0 * abs(float(E[n_, j])) + 1e-12)
    r = _check_recall(recall_case, _as_tensor(flipped["o"]), flipped["mask_out"])
    assert r.flips >= 1 and r.max_abs_rounded == 0.0


def test_recall_many_near_differences_are_all_forced():
    """A locality workload (4 x 32 x 32 tokens, 64 key tiles per row) at p = 0.9, where
    rows use up their skip budget, so many tiles sit near the boundary.  A stand-in
    kernel whose recall target is off by a hair (p * (1 + 1e-4)) decides differently
    at dozens of them; the harness must accept every such difference (each within the
    margin of the oracle run that follows the stand-in's earlier decisions) and
    compare the outputs against that run."""
    from temporal_block_sparse_sm_b200 import synthetic
    n_tok, dd = 4096, 64
    cfg = synthetic.WorkloadConfig("line", 1, 1, n_tok, dd, dd, dd, (4, 32, 32), 1, 0.05, 0.0)
    q, k, v = synthetic.Workload(cfg, seed=1, device="cpu").inputs(0)
    bits = lambda x: x.contiguous().view(torch.int16).numpy().view(np.uint16)
    qh, kh, vh = bits(q), bits(k), bits(v)
    tq, tk, _ = oracle.tiles(n_tok, dd, dd)
    items = np.arange(tq)
    full = oracle.all_live_rows(tq, n_tok, dd)
    p0 = 0.9
    base = oracle.step_recall(qh, kh, vh, B=1, H=1, N=n_tok, d=dd, Br=dd, Bc=dd, p=p0, items=items, mask_in=full)
    other = oracle.step_recall(qh, kh, vh, B=1, H=1, N=n_tok, d=dd, Br=dd, Bc=dd, p=p0 * (1 + 1e-4), items=items,
                               mask_in=full)
    n_diff = int((oracle.bits_to_bool(other["mask_out"], tk) != oracle.bits_to_bool(base["mask_out"], tk)).sum())
    assert n_diff >= 10, n_diff
    o = torch.from_numpy(other["o"].reshape(1, 1, tq * dd, dd)[:, :, :n_tok].copy()).to(torch.bfloat16)
    dummy = torch.empty(0)
    r = check_step(dummy, dummy, dummy, o, full, other["mask_out"], B=1, H=1, N=n_tok, d=dd, Br=dd, Bc=dd, p=p0,
                   items=items, host_qkv=(qh, kh, vh))
    assert r.flips >= 1 and r.max_abs_rounded == 0.0
