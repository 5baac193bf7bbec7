"""Pins for the CPU oracle (no GPU).

The oracle is checked against things other than itself:
  * library softmax attention (torch SDPA, fp64) when nothing can die, and
    restricted to the key tiles that stay live for any threshold;
  * a closed-form prefix-max statement of the decision;
  * a brute-force fixed-point characterisation over all subsets of tiles;
  * invariants (monotone masks, first tile live, monotone in tau, independent
    work items);
  * the analytic bound on the error that skipped tiles can cause, coarse (dead
    columns * e^tau) and per killed tile (width * e^{D_j});
  * the final running max and denominator against numpy max / exp-sum, and the
    exact split of the dense output into its live and skipped parts;
  * the hand-built fixtures in tests/golden/.
"""
from __future__ import annotations

import glob
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from tests.helpers import bf16_bits, bits_to_f64, random_qkv, sdpa_f64
from temporal_block_sparse_sm_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, tau, mask_in=None, force=None):
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    items = np.arange(B * H * Tq)
    if mask_in is None:
        mask_in = oracle_mod.all_live_rows(len(items), N, Bc)
    return items, mask_in, oracle_mod.step(q, k, v, B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, tau=tau,
                                           items=items, mask_in=mask_in, force=force)


def _gather_rows(o, B, H, N, Br):
    """oracle o [items, Br, d] -> [B, H, N, d] (drops rows past N)."""
    Tq = -(-N // Br)
    d = o.shape[-1]
    full = o.reshape(B, H, Tq * Br, d)[:, :, :N]
    return full


def _logits(q, k, d):
    qf = bits_to_f64(q)
    kf = bits_to_f64(k)
    return np.einsum("bhnd,bhmd->bhnm", qf, kf) / math.sqrt(d)


# --------------------------------------------------------------------------------------------
# 1. tau = -inf (nothing can die): equals library dense attention
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("N,d,Br,Bc", [(1, 64, 64, 64), (63, 64, 64, 64), (64, 64, 64, 64), (65, 64, 64, 64),
                                       (200, 64, 64, 64), (1024, 64, 64, 64), (200, 128, 128, 128),
                                       (1024, 128, 128, 128), (200, 64, 32, 48)])
def test_dense_limit_equals_library_attention(oracle_mod, N, d, Br, Bc):
    B, H = 1, 2
    q, k, v = random_qkv(B, H, N, d, seed=N * 7 + d)
    items, mask_in, res = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, -math.inf)
    ref = sdpa_f64(bits_to_f64(q), bits_to_f64(k), bits_to_f64(v))
    got = _gather_rows(res["o"], B, H, N, Br)
    err = np.abs(got - ref).max() / max(1.0, np.abs(ref).max())
    assert err <= 1e-12, err
    assert np.array_equal(res["mask_out"], mask_in)


def test_very_negative_finite_tau_equals_dense(oracle_mod):
    B, H, N, d = 1, 1, 300, 64
    q, k, v = random_qkv(B, H, N, d, seed=3)
    _, mask_in, res = _run_all_items(oracle_mod, q, k, v, B, H, N, d, 64, 64, -1e30)
    ref = sdpa_f64(bits_to_f64(q), bits_to_f64(k), bits_to_f64(v))
    assert np.abs(_gather_rows(res["o"], B, H, N, 64) - ref).max() <= 1e-12
    assert np.array_equal(res["mask_out"], mask_in)


# --------------------------------------------------------------------------------------------
# 2. any tau: the output is attention restricted to the key tiles that stay live
# --------------------------------------------------------------------------------------------
def _locality_inputs(N=320, d=64, H=2, seed=0, grid=(5, 8, 8)):
    cfg = synthetic.WorkloadConfig("t", 1, H, N, d, 64, 64, grid, 2, 0.05, 0.0)
    wl = synthetic.Workload(cfg, seed=seed)
    q, k, v = wl.inputs(0)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v)


@pytest.mark.parametrize("tau", [math.log(1e-2), math.log(1e-4), math.log(1e-8)])
@pytest.mark.parametrize("random_mask", [False, True])
def test_output_is_attention_over_live_out_tiles(oracle_mod, tau, random_mask):
    B, H, N, d, Br, Bc = 1, 2, 320, 64, 64, 64
    q, k, v = _locality_inputs(N, d, H)
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    mask_in = None
    if random_mask:
        rng = np.random.default_rng(5)
        live = rng.random((B * H * Tq, Tk)) < 0.7
        mask_in = oracle_mod.bool_to_bits(live)
    items, mask_in, res = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, tau, mask_in)
    live_out = oracle_mod.bits_to_bool(res["mask_out"], Tk)            # [items, Tk]
    qf, kf, vf = bits_to_f64(q), bits_to_f64(k), bits_to_f64(v)
    n_dead = 0
    for it in items:
        bh, i = divmod(int(it), Tq)
        b, h = divmod(bh, H)
        r0, r1 = i * Br, min(N, (i + 1) * Br)
        cols = np.repeat(live_out[it], Bc)[:N]
        n_dead += int((~live_out[it]).sum())
        if not cols.any():
            assert np.all(res["o"][it] == 0.0)
            continue
        mask = np.broadcast_to(cols, (r1 - r0, N))
        ref = sdpa_f64(qf[b, h, r0:r1], kf[b, h], vf[b, h], attn_mask=mask)
        assert np.abs(res["o"][it, : r1 - r0] - ref).max() <= 1e-12
    if tau > -5 and not random_mask:
        assert n_dead > 0, "the locality inputs should kill some tiles at this threshold"


# --------------------------------------------------------------------------------------------
# 3. the streaming decision equals a closed-form prefix-max rule
# --------------------------------------------------------------------------------------------
def _tile_maxima(s, N, Br, Bc, bh_i):
    """m_loc[j][r] for one item, plain numpy maxima over valid columns."""
    Tk = -(-N // Bc)
    return np.stack([s[:, j * Bc:min(N, (j + 1) * Bc)].max(axis=1) for j in range(Tk)])


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("tau", [-0.3, math.log(1e-2), math.log(1e-4)])
def test_decision_matches_closed_form(oracle_mod, seed, tau):
    B, H, N, d, Br, Bc = 1, 2, 300, 64, 64, 64
    q, k, v = _locality_inputs(N, d, H, seed=seed, grid=(3, 10, 10))
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    rng = np.random.default_rng(seed)
    live_in = rng.random((B * H * Tq, Tk)) < 0.8
    mask_in = oracle_mod.bool_to_bits(live_in)
    items, _, res = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, tau, mask_in)
    S = _logits(q, k, d)
    live_out = oracle_mod.bits_to_bool(res["mask_out"], Tk)
    for it in items:
        bh, i = divmod(int(it), Tq)
        s = S[0, bh, i * Br:min(N, (i + 1) * Br)]
        mloc = _tile_maxima(s, N, Br, Bc, it)
        L = np.flatnonzero(live_in[it])
        for j in range(Tk):
            if j not in L:
                assert math.isnan(res["D"][it, j]) and not live_out[it, j]
                continue
            earlier = [jj for jj in L if jj < j]
            if not earlier:
                expect = math.inf
            else:
                prefix = np.max(mloc[earlier], axis=0)
                expect = float(np.max(mloc[j] - prefix))
            got = res["D"][it, j]
            assert (got == expect) if math.isinf(expect) else abs(got - expect) <= 1e-12
            assert live_out[it, j] == (not (expect < tau) if abs(expect - tau) > 1e-9 else live_out[it, j])


# --------------------------------------------------------------------------------------------
# 4. brute force: the live-out set is the unique subset satisfying the fixed-point rule
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(6))
def test_live_set_is_unique_fixed_point(oracle_mod, seed):
    B, H, N, d, Br, Bc = 1, 1, 250, 64, 128, 64            # Tk = 4, Tq = 2
    q, k, v = random_qkv(B, H, N, d, seed=100 + seed, scale_qk=2.0)
    tau = [-0.5, -1.0, -2.0, -4.0, -8.0, -0.05][seed]
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    items, mask_in, res = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, tau)
    S = _logits(q, k, d)[0, 0]
    live_out = oracle_mod.bits_to_bool(res["mask_out"], Tk)
    for it in items:
        s = S[it * Br:min(N, (it + 1) * Br)]
        mloc = [s[:, j * Bc:min(N, (j + 1) * Bc)].max(axis=1) for j in range(Tk)]
        solutions = []
        for bits in itertools.product([False, True], repeat=Tk):
            ok = True
            for j in range(Tk):
                prev = [jj for jj in range(j) if bits[jj]]
                rise = math.inf if not prev else float(np.max(mloc[j] - np.max([mloc[p] for p in prev], axis=0)))
                if bits[j] != (rise >= tau):
                    ok = False
                    break
            if ok:
                solutions.append(bits)
        assert len(solutions) == 1
        assert tuple(live_out[it]) == solutions[0]


# --------------------------------------------------------------------------------------------
# 5. invariants
# --------------------------------------------------------------------------------------------
def test_masks_monotone_and_first_live_tile_kept(oracle_mod):
    B, H, N, d, Br, Bc = 1, 2, 320, 64, 64, 64
    q, k, v = _locality_inputs(N, d, H, seed=4)
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    rng = np.random.default_rng(1)
    live_in = rng.random((B * H * Tq, Tk)) < 0.6
    mask_in = oracle_mod.bool_to_bits(live_in)
    _, _, res = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, math.log(1e-2), mask_in)
    live_out = oracle_mod.bits_to_bool(res["mask_out"], Tk)
    assert not np.any(live_out & ~live_in)
    for it in range(live_in.shape[0]):
        idx = np.flatnonzero(live_in[it])
        if idx.size:
            assert live_out[it, idx[0]]
            assert res["D"][it, idx[0]] == math.inf


def test_dead_set_grows_with_tau(oracle_mod):
    B, H, N, d, Br, Bc = 1, 2, 320, 64, 64, 64
    q, k, v = _locality_inputs(N, d, H, seed=7)
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    prev_live = None
    for tau in [-math.inf, math.log(1e-8), math.log(1e-5), math.log(1e-4), math.log(1e-3), math.log(1e-2), -0.1]:
        _, _, res = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, tau)
        live = oracle_mod.bits_to_bool(res["mask_out"], Tk)
        if prev_live is not None:
            assert not np.any(live & ~prev_live)
        prev_live = live
    assert (~prev_live).sum() > 0


def test_work_items_are_independent(oracle_mod):
    N, d, Br, Bc, tau = 192, 64, 64, 64, math.log(1e-3)
    q2, k2, v2 = random_qkv(2, 3, N, d, seed=11, scale_qk=2.0)
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    items2, _, res2 = _run_all_items(oracle_mod, q2, k2, v2, 2, 3, N, d, Br, Bc, tau)
    # a B=2 run equals two B=1 runs
    for b in range(2):
        _, _, r1 = _run_all_items(oracle_mod, q2[b:b + 1], k2[b:b + 1], v2[b:b + 1], 1, 3, N, d, Br, Bc, tau)
        sl = slice(b * 3 * Tq, (b + 1) * 3 * Tq)
        assert np.array_equal(r1["o"], res2["o"][sl])
        assert np.array_equal(r1["mask_out"], res2["mask_out"][sl])
    # permuting heads permutes the outputs
    perm = [2, 0, 1]
    _, _, rp = _run_all_items(oracle_mod, q2[:, perm], k2[:, perm], v2[:, perm], 2, 3, N, d, Br, Bc, tau)
    o2 = res2["o"].reshape(2, 3, Tq, Br, d)
    op = rp["o"].reshape(2, 3, Tq, Br, d)
    assert np.array_equal(op, o2[:, perm])
    # running a subset of items gives the same rows as the full run
    sub = np.array([5, 0, 17, 9])
    rs = oracle_mod.step(q2, k2, v2, B=2, H=3, N=N, d=d, Br=Br, Bc=Bc, tau=tau, items=sub,
                         mask_in=oracle_mod.all_live_rows(len(sub), N, Bc))
    assert np.array_equal(rs["o"], res2["o"][sub])
    assert np.array_equal(rs["mask_out"], res2["mask_out"][sub])


def test_forced_decisions(oracle_mod):
    B, H, N, d, Br, Bc = 1, 1, 256, 64, 64, 64
    q, k, v = _locality_inputs(N, d, H, seed=2, grid=(4, 8, 8))
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    items, mask_in, own = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, math.log(1e-2))
    # forcing the oracle's own decisions changes nothing
    live = oracle_mod.bits_to_bool(own["mask_out"], Tk)
    forced = np.where(live, 1, 0).astype(np.int8)
    _, _, same = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, math.log(1e-2), force=forced)
    assert np.array_equal(same["o"], own["o"]) and np.array_equal(same["mask_out"], own["mask_out"])
    # forcing everything live gives dense attention
    _, _, dense = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, math.log(1e-2),
                                 force=np.ones((len(items), Tk), np.int8))
    ref = sdpa_f64(bits_to_f64(q), bits_to_f64(k), bits_to_f64(v))
    assert np.abs(_gather_rows(dense["o"], B, H, N, Br) - ref).max() <= 1e-12


def test_invalid_arguments_rejected(oracle_mod):
    q, k, v = random_qkv(1, 1, 64, 64, seed=0)
    with pytest.raises(ValueError):
        oracle_mod.step(q, k, v, B=1, H=1, N=64, d=64, Br=64, Bc=64, tau=0.5, items=[0],
                        mask_in=oracle_mod.all_live_rows(1, 64, 64))
    with pytest.raises(ValueError):
        oracle_mod.step(q, k, v, B=1, H=1, N=64, d=64, Br=64, Bc=64, tau=float("nan"), items=[0],
                        mask_in=oracle_mod.all_live_rows(1, 64, 64))
    with pytest.raises(ValueError):
        oracle_mod.step(q, k, v, B=1, H=1, N=64, d=64, Br=64, Bc=64, tau=-1.0, items=[1],
                        mask_in=oracle_mod.all_live_rows(1, 64, 64))


# --------------------------------------------------------------------------------------------
# 6. error bound: skipped mass is at most (#dead columns) * exp(tau)
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("tau", list(synthetic.CONFIGS["c5"].fixed_taus))
def test_error_bound_vs_dense(oracle_mod, tau):
    B, H, N, d, Br, Bc = 1, 2, 512, 64, 64, 64
    q, k, v = _locality_inputs(N, d, H, seed=9, grid=(2, 16, 16))
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    items, mask_in, res = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, tau)
    qf, kf, vf = bits_to_f64(q), bits_to_f64(k), bits_to_f64(v)
    dense = sdpa_f64(qf, kf, vf)
    live_out = oracle_mod.bits_to_bool(res["mask_out"], Tk)
    got = _gather_rows(res["o"], B, H, N, Br)
    for it in items:
        bh, i = divmod(int(it), Tq)
        r0, r1 = i * Br, min(N, (i + 1) * Br)
        dead_cols = sum(min(N, (j + 1) * Bc) - j * Bc for j in range(Tk) if not live_out[it, j])
        vrange = vf[0, bh].max(axis=0) - vf[0, bh].min(axis=0)
        bound = min(1.0, dead_cols * math.exp(tau)) * vrange
        err = np.abs(got[0, bh, r0:r1] - dense[0, bh, r0:r1])
        assert np.all(err <= bound[None, :] + 1e-12)
        if tau == -math.inf:
            assert dead_cols == 0


@pytest.mark.parametrize("tau", [math.log(0.5), math.log(1e-1), math.log(1e-2)])
def test_final_max_sum_and_per_tile_bound(oracle_mod, tau):
    """The oracle's final running max and denominator are numpy's max and sum of
    exponentials over the live-out columns.  The dense output splits exactly into
    the live part and the skipped part.  Each row's skipped mass (in units of its
    final max) is at most sum over killed tiles of width * e^{D_j}.  Killed entries
    satisfy s <= m_loc <= m_run + D_j <= m_fin + D_j.  That sum is itself below
    the coarse (dead columns) * e^tau bound."""
    B, H, N, d, Br, Bc = 1, 2, 512, 64, 64, 64
    q, k, v = _locality_inputs(N, d, H, seed=9, grid=(2, 16, 16))
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    items, mask_in, res = _run_all_items(oracle_mod, q, k, v, B, H, N, d, Br, Bc, tau)
    logits = _logits(q, k, d)
    qf, kf, vf = bits_to_f64(q), bits_to_f64(k), bits_to_f64(v)
    dense = sdpa_f64(qf, kf, vf)
    live_out = oracle_mod.bits_to_bool(res["mask_out"], Tk)
    n_killed = 0
    for it in items:
        bh, i = divmod(int(it), Tq)
        r0, r1 = i * Br, min(N, (i + 1) * Br)
        nr = r1 - r0
        cols = np.repeat(live_out[it], Bc)[:N]
        s = logits[0, bh, r0:r1]
        m = s[:, cols].max(axis=1)
        l = np.exp(s[:, cols] - m[:, None]).sum(axis=1)
        np.testing.assert_allclose(res["m_fin"][it, :nr], m, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(res["l_fin"][it, :nr], l, rtol=1e-12)
        assert np.all(res["l_fin"][it, :nr] >= 1.0 - 1e-15)           # the row max is in a live tile
        assert np.all(np.isnan(res["m_fin"][it, nr:])) and np.all(np.isnan(res["l_fin"][it, nr:]))
        w = np.exp(s[:, ~cols] - m[:, None])                          # skipped weights
        S = w.sum(axis=1)
        o_sparse = res["o"][it, :nr]
        recon = (l[:, None] * o_sparse + w @ vf[0, bh][~cols]) / (l + S)[:, None]
        np.testing.assert_allclose(recon, dense[0, bh, r0:r1], rtol=0, atol=1e-12)
        killed = [j for j in range(Tk) if not live_out[it, j]]         # mask_in is all-live: every tile was tested
        n_killed += len(killed)
        assert all(res["D"][it, j] < tau for j in killed)
        widths = [min(N, (j + 1) * Bc) - j * Bc for j in killed]
        sharp = sum(wd * math.exp(res["D"][it, j]) for wd, j in zip(widths, killed))
        assert np.all(S <= sharp * (1 + 1e-12))
        assert sharp <= sum(widths) * math.exp(tau) * (1 + 1e-12)
        vrange = vf[0, bh].max(axis=0) - vf[0, bh].min(axis=0)
        err = np.abs(o_sparse - dense[0, bh, r0:r1])
        assert np.all(err <= min(1.0, sharp) * vrange[None, :] + 1e-12)
    assert n_killed > 0, "the case must kill tiles"


# --------------------------------------------------------------------------------------------
# 7. hand-built fixtures
# --------------------------------------------------------------------------------------------
def _expand(spec, n):
    out = np.full(n, float(spec.get("default", 0.0)))
    if "odd" in spec:
        out[1::2] = float(spec["odd"])
    for key, val in spec.get("set", {}).items():
        out[int(key)] = float(val)
    return out


def _load_fixture(path):
    with open(path) as f:
        fx = json.load(f)
    N, d = fx["N"], fx["d"]
    assert d == 64
    a, x = _expand(fx["a"], N), _expand(fx["x"], N)
    q = torch.zeros(1, 1, N, d)
    k = torch.zeros(1, 1, N, d)
    v = torch.zeros(1, 1, N, d)
    q[0, 0, :, 0] = torch.from_numpy(8.0 * a)
    k[0, 0, :, 0] = torch.from_numpy(x)
    v[0, 0, :, 0] = torch.from_numpy(_expand(fx["v0"], N))
    v[0, 0, :, 1] = torch.from_numpy(_expand(fx["v1"], N))
    for t in (q, k, v):
        assert torch.equal(t.to(torch.bfloat16).float(), t), "fixture values must be exact in bf16"
    return fx, bf16_bits(q), bf16_bits(k), bf16_bits(v)


FIXTURES = sorted(glob.glob(os.path.join(GOLDEN, "*.json")))


@pytest.mark.parametrize("path", FIXTURES, ids=[os.path.basename(p) for p in FIXTURES])
def test_golden_fixture(oracle_mod, path):
    fx, q, k, v = _load_fixture(path)
    N, d, Br, Bc = fx["N"], fx["d"], fx["Br"], fx["Bc"]
    Tq, Tk, W = oracle_mod.tiles(N, Br, Bc)
    mask_in = None
    if fx["mask_in"] is not None:
        live = np.zeros((Tq, Tk), bool)
        for i, js in enumerate(fx["mask_in"]):
            live[i, js] = True
        mask_in = oracle_mod.bool_to_bits(live)
    items, mask_in, res = _run_all_items(oracle_mod, q, k, v, 1, 1, N, d, Br, Bc, fx["tau"], mask_in)
    live_out = oracle_mod.bits_to_bool(res["mask_out"], Tk)
    exp = fx["expect"]
    for i in range(Tq):
        assert list(np.flatnonzero(live_out[i])) == exp["mask_out"][i], (i, live_out[i])
        for j, e in enumerate(exp["D"][i]):
            got = res["D"][i, j]
            if e is None:
                assert math.isnan(got)
            elif e == "inf":
                assert got == math.inf
            else:
                assert abs(got - float(e)) <= 1e-12, (i, j, got, e)
        nr = min(Br, N - i * Br)
        for comp, key in ((0, "o0"), (1, "o1")):
            if key in exp:
                assert np.abs(res["o"][i, :nr, comp] - exp[key][i]).max() <= 1e-12
