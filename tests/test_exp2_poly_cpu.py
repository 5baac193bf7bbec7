"""The FMA-pipe exp2 of the softmax (CPU, no GPU).

Part of the attention kernel's exponentials skip MUFU.  They compute
2^x = 2^r * p(f), with r = round(x) and f = x - r in [-1/2, 1/2].  This is
Cody and Waite's range reduction.  p is the degree-3 minimax polynomial for
relative error, fitted by temporal_block_sparse_sm_b200/exp2_poly.py with the
Remez exchange algorithm.  Here:
  * refitting reproduces the kernel's fp32 constants (read from
    csrc/sm100_ptx.cuh);
  * those fp32 constants keep the relative error of p against 2^f on
    [-1/2, 1/2] at the documented 7.5e-5;
  * a numpy emulation of the device steps gives 2^x within that bound on
    [-125, 0] and at most 2^-125 below it.  The steps are fp32 rounding by
    the 1.5 * 2^23 constant, three fused multiply-adds, and r added into the
    exponent field.
The device code itself is checked against the same bound by the checked
build (tests/debug_build_checks.py).
"""
from __future__ import annotations

import os
import re

import numpy as np

from temporal_block_sparse_sm_b200 import exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "temporal_block_sparse_sm_b200", "csrc", "sm100_ptx.cuh")


def _kernel_constants() -> np.ndarray:
    text = open(PTX).read()
    vals = dict(re.findall(r"kExp2Poly(\d)\s*=\s*([-+0-9.eE]+)f;", text))
    assert sorted(vals) == ["0", "1", "2", "3"], vals
    return np.array([float(vals[str(i)]) for i in range(4)], dtype=np.float32)


def test_refit_reproduces_the_kernel_constants():
    coef, err64 = exp2_poly.remez_exp2()
    c32 = coef.astype(np.float32)
    k = _kernel_constants()
    assert np.all(np.abs(c32 - k) <= np.spacing(np.abs(k))), (c32, k)
    assert err64 <= 7.5e-5


def test_fp32_constants_meet_the_bound():
    k = _kernel_constants().astype(np.float64)
    f = np.linspace(-0.5, 0.5, 400001)
    rel = np.abs(np.polyval(k[::-1], f) / np.exp2(f) - 1.0).max()
    assert rel <= 7.55e-5, rel


def _emulate(x: np.ndarray) -> np.ndarray:
    """The device steps in fp32 (fused multiply-add as one fp64 step, then rounded)."""
    k = _kernel_constants()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)                       # 1.5 * 2^23
    t = (x + magic).astype(np.float32)                   # round(x) in the low mantissa bits
    f = (x - (t - magic)).astype(np.float32)

    def fma(a, b, c):
        return (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)

    q = fma(np.full_like(f, k[3]), f, k[2])
    q = fma(q, f, k[1])
    q = fma(q, f, k[0])
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_emulated_device_steps_stay_within_the_bound():
    x = np.concatenate([np.linspace(-125.0, 0.0, 1 << 20), [0.0, -1e-7, -0.5, -0.50000006, -124.5, -125.0]])
    x = x.astype(np.float32)
    y = _emulate(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0).max()
    assert rel <= 7.6e-5, rel
    low = _emulate(np.array([-125.5, -126.0, -130.0, -1000.0, -np.inf], dtype=np.float32)).astype(np.float64)
    assert np.all(np.isfinite(low)) and np.all(low >= 0.0) and np.all(low <= 2.0 ** -125)
