"""Pins of the fixed-recall ("cumulative energy") oracle, ``oracle.step_recall`` (CPU).

Page: "Training-free sparse attention based on cumulative energy filtering"
(abstract): keep a fixed recall rate of the attention mass, with a dynamic
threshold, inside the FlashAttention pass.  The oracle's reading is written at
the top of ``oracle/recall_oracle.c``.  Nothing here retypes its update rule;
each pin is a fact that any correct implementation of that reading must show:

1. p = 1 affords no skipped mass: the step is dense softmax attention (library
   routine), partial tiles included.
2. The output is softmax attention restricted to the keys of the tiles the
   step kept (library routine with a boolean mask).
3. Recall floor: for every valid query row, the softmax mass of its kept keys
   over the mass of all keys it was offered (tiles live in mask_in), computed
   here from scratch, is at least p.  The predicate must also skip something
   at moderate p (it is not vacuous).
4. Tiles of constant logits carry exactly the mass bound the predicate uses,
   so there the decision is closed-form: walking the tiles in ascending order,
   a tile is skipped exactly when the row's recall, counting it with the tiles
   already skipped, stays at least p.  Worked cases with hand-derived
   boundaries, and a brute-force walk over random constant-tile rows.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import bits_to_f64, random_qkv, sdpa_f64


def _all_items(B, H, N, Br):
    return np.arange(B * H * -(-N // Br))


def _rows(res_o, B, H, N, Br):
    """[items, Br, d] -> [B, H, N, d] (drop rows past N)."""
    Tq = -(-N // Br)
    d = res_o.shape[-1]
    return res_o.reshape(B, H, Tq * Br, d)[:, :, :N]


def _tile_scaled_qkv(B, H, N, d, Bc, seed, scales):
    """Random q, k, v with key tiles at different scales, so that weak tiles fall
    far below the running max (bf16 bit patterns)."""
    g = torch.Generator().manual_seed(seed)
    q = 2.0 * torch.randn(B, H, N, d, generator=g)
    k = 2.0 * torch.randn(B, H, N, d, generator=g)
    for j in range(-(-N // Bc)):
        k[:, :, j * Bc:(j + 1) * Bc] *= scales[j % len(scales)]
    v = torch.randn(B, H, N, d, generator=g)
    to = lambda x: x.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)
    return to(q), to(k), to(v)


def _live_cols(bits_rows, N, Br, Bc, B, H):
    """[B, H, N(query), N(key)] bool: key column c is in a tile live in the query row's mask row."""
    Tq, Tk, W = oracle.tiles(N, Br, Bc)
    live = oracle.bits_to_bool(bits_rows, Tk).reshape(B, H, Tq, Tk)
    cols = np.repeat(live, Bc, axis=3)[..., :N]          # [B, H, Tq, N]
    return np.repeat(cols, Br, axis=2)[:, :, :N]          # [B, H, N, N]


# ------------------------------------------------------------------------------------------ 1
@pytest.mark.parametrize("N,d,Br,Bc", [(1, 64, 64, 64), (63, 64, 64, 64), (65, 64, 64, 64), (200, 64, 64, 64),
                                       (300, 128, 128, 128), (200, 64, 32, 48)])
def test_recall_one_is_dense_attention(oracle_mod, N, d, Br, Bc):
    B, H = 1, 2
    q, k, v = random_qkv(B, H, N, d, seed=N + 3 * d, scale_qk=2.0)
    items = _all_items(B, H, N, Br)
    full = oracle.all_live_rows(len(items), N, Bc)
    res = oracle.step_recall(q, k, v, B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, p=1.0, items=items, mask_in=full)
    assert np.array_equal(res["mask_out"], full)
    ref = sdpa_f64(bits_to_f64(q), bits_to_f64(k), bits_to_f64(v))
    assert np.abs(_rows(res["o"], B, H, N, Br) - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


# ------------------------------------------------------------------------------------------ 2, 3
@pytest.mark.parametrize("p", [0.5, 0.9, 0.99, 0.999])
@pytest.mark.parametrize("N,d,Br,Bc,live_frac", [(300, 64, 64, 64, 1.0), (300, 64, 64, 64, 0.7),
                                                 (520, 128, 128, 128, 1.0), (200, 64, 32, 48, 0.8)])
def test_output_is_attention_over_kept_keys_and_recall_holds(oracle_mod, p, N, d, Br, Bc, live_frac):
    B, H = 1, 2
    q, k, v = _tile_scaled_qkv(B, H, N, d, Bc, seed=int(p * 1000) + N, scales=[1.0, 0.3, 0.8, 0.15, 0.5])
    items = _all_items(B, H, N, Br)
    Tq, Tk, W = oracle.tiles(N, Br, Bc)
    rng = np.random.default_rng(N + d)
    live = rng.random((len(items), Tk)) < live_frac
    live[:, 0] = True
    bits_in = oracle.bool_to_bits(live)
    res = oracle.step_recall(q, k, v, B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, p=p, items=items, mask_in=bits_in)
    kept = oracle.bits_to_bool(res["mask_out"], Tk)
    assert not (kept & ~live).any(), "a tile dead on entry came back"
    qf, kf, vf = bits_to_f64(q), bits_to_f64(k), bits_to_f64(v)
    # 2: the output is library attention over the kept keys (rows with nothing kept are 0)
    kept_cols = _live_cols(res["mask_out"], N, Br, Bc, B, H)
    any_kept = kept_cols.any(-1, keepdims=True)
    ref = sdpa_f64(qf, kf, vf, attn_mask=np.where(any_kept, kept_cols, True))
    ref = np.where(any_kept, ref, 0.0)
    assert np.abs(_rows(res["o"], B, H, N, Br) - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    # 3: recall floor per valid row, from softmax probabilities over the offered keys
    offered = _live_cols(bits_in, N, Br, Bc, B, H)
    s = np.einsum("bhnd,bhmd->bhnm", qf, kf) / math.sqrt(d)
    s = np.where(offered, s, -np.inf)
    w = np.exp(s - s.max(-1, keepdims=True))
    recall = (w * kept_cols).sum(-1) / w.sum(-1)
    assert recall.min() >= p - 1e-12, (recall.min(), p)
    if p <= 0.9:
        assert (live & ~kept).sum() > 0, "the predicate should skip tiles at this recall"


def test_recall_floor_on_locality_inputs(oracle_mod):
    """The c1 locality workload at p = 0.95: every row keeps >= 95% of its mass,
    and tiles are skipped.  The mass bound of a tile (its width times its peak
    weight) is loose, so the realised recall sits well above the floor."""
    from temporal_block_sparse_sm_b200 import synthetic
    cfg = synthetic.CONFIGS["c1"]
    q, k, v = synthetic.Workload(cfg, seed=0, device="cpu").inputs(0)
    to = lambda x: x.contiguous().view(torch.int16).numpy().view(np.uint16)
    qh, kh, vh = to(q), to(k), to(v)
    B, H, N, d, Br, Bc = cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc
    items = _all_items(B, H, N, Br)
    full = oracle.all_live_rows(len(items), N, Bc)
    p = 0.95
    res = oracle.step_recall(qh, kh, vh, B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, p=p, items=items, mask_in=full)
    kept_cols = _live_cols(res["mask_out"], N, Br, Bc, B, H)
    qf, kf = bits_to_f64(qh), bits_to_f64(kh)
    s = np.einsum("bhnd,bhmd->bhnm", qf, kf) / math.sqrt(d)
    w = np.exp(s - s.max(-1, keepdims=True))
    recall = (w * kept_cols).sum(-1) / w.sum(-1)
    assert recall.min() >= p - 1e-12
    Tk = -(-N // Bc)
    skipped = 1.0 - oracle.bits_to_bool(res["mask_out"], Tk).mean()
    assert skipped > 0.05, skipped
    assert recall.mean() > p
    # the reported bounds: l / (l + z) >= p for every row, and z covers the true skipped mass
    l, z = res["l_fin"], res["z_fin"]
    assert (l / (l + z) >= p - 1e-12).all()


# ------------------------------------------------------------------------------------------ 4
def _constant_tile_case(tile_logits, widths, d=64, Bc=64):
    """One query row block whose logit against every key of tile j is tile_logits[j]
    (exact in bf16): q rows = a * e0, keys of tile j = (tile_logits[j] * sqrt(d) / a) * e0."""
    N = sum(widths)
    assert all(wd == Bc for wd in widths[:-1]) and 1 <= widths[-1] <= Bc
    a = 8.0
    q = np.zeros((1, 1, N, d), np.float32)
    k = np.zeros((1, 1, N, d), np.float32)
    q[..., 0] = a
    c0 = 0
    for t, wd in zip(tile_logits, widths):
        k[0, 0, c0:c0 + wd, 0] = t * math.sqrt(d) / a
        c0 += wd
    v = np.random.default_rng(len(widths)).standard_normal((1, 1, N, d)).astype(np.float32)
    to = lambda x: torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    qb, kb, vb = to(q), to(k), to(v)
    # the logits the oracle sees (bf16-rounded keys)
    kt = bits_to_f64(kb)[0, 0, :, 0]
    logits = [float(a * kt[sum(widths[:j])] / math.sqrt(d)) for j in range(len(widths))]
    return qb, kb, vb, N, logits


def _expected_by_prefix_recall(logits, widths, p):
    """Closed form for constant tiles: walk the tiles in order; skip a tile when the
    recall (kept mass / (kept + skipped mass), over the tiles seen so far and this
    one) would stay >= p.  The first tile is always kept."""
    kept, skipped, out = 0.0, 0.0, []
    for j, (s, wd) in enumerate(zip(logits, widths)):
        m = wd * math.exp(s)
        if j > 0 and kept / (kept + skipped + m) >= p:
            skipped += m
            out.append(False)
        else:
            kept += m
            out.append(True)
    return out


@pytest.mark.parametrize("logits,widths,p,live", [
    # two full tiles, logits 0 and b, p = 0.9: skip tile 1 iff e^b / (1 + e^b) <= 0.1, i.e. b <= -ln 9 = -2.197
    ([0.0, -2.0], [64, 64], 0.9, [1, 1]), ([0.0, -2.5], [64, 64], 0.9, [1, 0]),
    # second tile 36 keys wide: skip iff 36 e^b <= 64 / 9, i.e. b <= ln(64 / 324) = -1.622
    ([0.0, -1.5], [64, 36], 0.9, [1, 1]), ([0.0, -1.75], [64, 36], 0.9, [1, 0]),
    # p = 0.99: skip iff e^b <= 1/99, b <= -4.595
    ([0.0, -4.4], [64, 64], 0.99, [1, 1]), ([0.0, -4.8], [64, 64], 0.99, [1, 0]),
    # a tile above the running max can never be afforded
    ([0.0, 0.5], [64, 64], 0.5, [1, 1]),
    # skipped mass accumulates: after tile 1 (mass 64 e^-2.5 = 5.25) is skipped, tile 2 fits
    # only while 5.25 + 64 e^b <= 64 / 9, i.e. b <= -3.539 (recall 64 / (64 + 5.25 + 64 e^b) >= 0.9)
    ([0.0, -2.5, -3.4], [64, 64, 64], 0.9, [1, 0, 1]), ([0.0, -2.5, -3.7], [64, 64, 64], 0.9, [1, 0, 0]),
    # the running max rises after a skip: tile 1 (64 e^-3) is skipped, tile 2 (logit 1) is kept;
    # tile 3 is then skipped iff recall (64 + 64 e) / (64 + 64 e + 64 e^-3 + 64 e^b) >= 0.9, i.e. b <= -1.012
    ([0.0, -3.0, 1.0, -1.15], [64, 64, 64, 64], 0.9, [1, 0, 1, 0]),
    ([0.0, -3.0, 1.0, -0.9], [64, 64, 64, 64], 0.9, [1, 0, 1, 1]),
])
def test_worked_cases(oracle_mod, logits, widths, p, live):
    q, k, v, N, actual = _constant_tile_case(logits, widths)
    Tk = len(widths)
    Tq = -(-N // 64)
    res = oracle.step_recall(q, k, v, B=1, H=1, N=N, d=64, Br=64, Bc=64, p=p, items=np.arange(Tq),
                             mask_in=oracle.all_live_rows(Tq, N, 64))
    got = oracle.bits_to_bool(res["mask_out"], Tk)
    assert _expected_by_prefix_recall(actual, widths, p) == [bool(x) for x in live], actual
    for j in range(Tk):
        assert (got[:, j] == bool(live[j])).all(), (actual, got)


def test_constant_tiles_brute_force(oracle_mod):
    """Random rows of 2..6 constant tiles against the prefix-recall walk."""
    rng = np.random.default_rng(5)
    n_cases = 0
    for case in range(60):
        T = int(rng.integers(2, 7))
        widths = [64] * (T - 1) + [int(rng.integers(1, 65))]
        tl = [0.0] + list(rng.uniform(-9.0, 0.5, size=T - 1))
        p = float(rng.choice([0.5, 0.8, 0.9, 0.99]))
        q, k, v, N, logits = _constant_tile_case(tl, widths)
        want = _expected_by_prefix_recall(logits, widths, p)
        res = oracle.step_recall(q, k, v, B=1, H=1, N=N, d=64, Br=64, Bc=64, p=p, items=np.arange(-(-N // 64)),
                                 mask_in=oracle.all_live_rows(-(-N // 64), N, 64))
        E = res["E"]
        # skip a case whose decision sits at rounding distance of the boundary
        if np.nanmin(np.abs(E[np.isfinite(E)])) < 1e-9 if np.isfinite(E).any() else False:
            continue
        got = oracle.bits_to_bool(res["mask_out"], T)
        assert all((got[:, j] == want[j]).all() for j in range(T)), (tl, widths, p, want, got)
        n_cases += 1
    assert n_cases >= 50


def test_p_out_of_range_is_rejected(oracle_mod):
    q, k, v = random_qkv(1, 1, 64, 64, seed=1)
    for p in (0.0, -0.1, 1.5, float("nan")):
        with pytest.raises(ValueError):
            oracle.step_recall(q, k, v, B=1, H=1, N=64, d=64, Br=64, Bc=64, p=p, items=np.arange(1),
                               mask_in=oracle.all_live_rows(1, 64, 64))
