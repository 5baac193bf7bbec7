"""GPU-vs-oracle parity harness (used by the -m gpu tests and smoke()).

Teacher forcing: for every checked step the oracle receives the GPU's own
incoming mask rows, so a decision that sits within rounding distance of the
threshold cannot compound across steps.

Acceptance (bf16 inputs, fp32 accumulation on the GPU, fp64 oracle):
  * masks: bit-exact, except tiles whose oracle margin |D_j - tau| is below
    MARGIN (natural log); those are counted and the oracle is re-run with the
    GPU's decision forced for them, so the output check covers arithmetic only;
  * outputs: max e <= MAX_ABS and mean e <= MEAN_ABS over the checked rows,
    with e = |o_gpu - o_oracle| / max(1, |o_oracle|): absolute for |o| <= 1,
    relative above.  A bf16 output of magnitude in [1, 2) is only stored to
    2^-8, and P enters P.V as bf16 (relative 2^-9 per weight), so an absolute
    1e-2 bound on outputs beyond 1 would test the storage format, not the
    kernel.  The absolute maximum is reported as well.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np
import torch

import oracle
from tests.helpers import bf16_bits

MARGIN = 1e-3
MAX_ABS = 1e-2
MEAN_ABS = 1e-3


@dataclass
class StepCheck:
    step: int
    tau: float
    n_items: int
    tiles_tested: int
    flips: int
    max_abs: float
    mean_abs: float
    max_abs_rounded: float
    skip_fraction: float
    max_abs_unscaled: float = 0.0
    notes: List[str] = field(default_factory=list)


def pick_items(B: int, H: int, Tq: int, n: int, seed: int) -> np.ndarray:
    """n work items (b*H+h)*Tq+i drawn by seed, always including i=0 and i=Tq-1 of some head."""
    R = B * H * Tq
    if n >= R:
        return np.arange(R)
    rng = np.random.default_rng(seed)
    must = {0, Tq - 1, R - 1, R - Tq}
    rest = rng.choice(R, size=n, replace=False)
    out = list(dict.fromkeys([x for x in must if 0 <= x < R] + list(rest)))[:max(n, len(must))]
    return np.array(sorted(out), dtype=np.int64)


def gpu_rows(o: torch.Tensor, items: np.ndarray, N: int, Br: int, Tq: int, H: int) -> np.ndarray:
    """[n_items, Br, d] float64 rows of o for the items (rows past N are zero)."""
    d = o.shape[-1]
    out = np.zeros((len(items), Br, d), dtype=np.float64)
    of = o.detach()
    for n_, it in enumerate(items):
        bh, i = divmod(int(it), Tq)
        b, h = divmod(bh, H)
        r0, r1 = i * Br, min(N, (i + 1) * Br)
        out[n_, : r1 - r0] = of[b, h, r0:r1].float().cpu().numpy()
    return out


def check_step(q, k, v, o, bits_in: np.ndarray, bits_out: np.ndarray, *, B, H, N, d, Br, Bc, tau: float,
               items: np.ndarray, step: int = 0, threads: int = 0, host_qkv=None,
               max_abs: float = MAX_ABS, mean_abs: float = MEAN_ABS, relative_above_one: bool = True) -> StepCheck:
    Tq, Tk, W = oracle.tiles(N, Br, Bc)
    qh, kh, vh = host_qkv if host_qkv is not None else (bf16_bits(q), bf16_bits(k), bf16_bits(v))
    min_rows = bits_in[items]
    res = oracle.step(qh, kh, vh, B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, tau=tau, items=items, mask_in=min_rows,
                      threads=threads)
    g_live = oracle.bits_to_bool(bits_out[items], Tk)
    o_live = oracle.bits_to_bool(res["mask_out"], Tk)
    tested = ~np.isnan(res["D"])
    diff = g_live != o_live
    margin = np.abs(res["D"] - tau)
    near = tested & (margin < MARGIN)
    bad = diff & ~near
    assert not bad.any(), (f"step {step}: {int(bad.sum())} mask bits differ outside the margin; first at "
                           f"{np.argwhere(bad)[:5].tolist()}, margins {margin[bad][:5]}")
    # dead-on-entry tiles must stay dead, bits past Tk must be 0
    in_live = oracle.bits_to_bool(min_rows, Tk)
    assert not (g_live & ~in_live).any(), "GPU revived a tile that was dead on entry"
    flips = int((diff & near).sum())
    ref_o = res["o"]
    if flips:
        rows = np.flatnonzero((diff & near).any(axis=1))
        force = np.where(tested[rows], g_live[rows].astype(np.int8), np.int8(-1)).astype(np.int8)
        res2 = oracle.step(qh, kh, vh, B=B, H=H, N=N, d=d, Br=Br, Bc=Bc, tau=tau, items=items[rows],
                           mask_in=min_rows[rows], force=force, threads=threads)
        ref_o = ref_o.copy()
        ref_o[rows] = res2["o"]
    got = gpu_rows(o, items, N, Br, Tq, H)
    valid = np.zeros((len(items), Br), dtype=bool)
    for n_, it in enumerate(items):
        i = int(it) % Tq
        valid[n_, : min(Br, N - i * Br)] = True
    err_abs = np.abs(got - ref_o)
    err = err_abs / np.maximum(1.0, np.abs(ref_o)) if relative_above_one else err_abs
    err = err[valid]
    mx_abs = float(err_abs[valid].max())
    rounded = torch.from_numpy(ref_o).to(torch.bfloat16).double().numpy()
    err_r = np.abs(got - rounded)[valid]
    mx, mn = float(err.max()), float(err.mean())
    assert np.isfinite(got[valid]).all(), "non-finite outputs"
    assert mx <= max_abs, f"step {step}: max error = {mx} (absolute {mx_abs})"
    assert mn <= mean_abs, f"step {step}: mean error = {mn}"
    return StepCheck(step, tau, len(items), int(tested.sum()), flips, mx, mn, float(err_r.max()),
                     1.0 - float(g_live.mean()), mx_abs)
