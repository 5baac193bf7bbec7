"""Coefficients of the FMA-pipe exp2 used for part of the softmax exponentials.

2^x is evaluated as 2^r * p(f) with r = round(x), f = x - r in [-1/2, 1/2]
(Cody and Waite's range reduction), and p the degree-3 polynomial that
minimises the maximum *relative* error of p(f) against 2^f on [-1/2, 1/2],
found here with the Remez exchange algorithm.  Run this file to reproduce
the constants in csrc/sm100_ptx.cuh (kExp2Poly*).
"""
from __future__ import annotations

import numpy as np


def remez_exp2(degree: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 50):
    n = degree + 2
    # Chebyshev extrema as the starting reference
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E * 2^x_i  (equioscillating relative error)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, : degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, -1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        coef = sol[: degree + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of the error, one per sign change interval
        sign = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if sign[i] != sign[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) >= n:
            # keep the n points with the largest error that still alternate
            while len(idx) > n:
                drop = 0 if abs(err[idx[0]]) < abs(err[idx[-1]]) else len(idx) - 1
                idx.pop(drop)
            x = grid[idx]
    err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
    return coef, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_exp2()
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 200001)
    e32 = np.abs((np.polyval(c32.astype(np.float64)[::-1], g) - 2.0 ** g) / 2.0 ** g).max()
    print("coefficients c0..c3 (float32):", [float(v) for v in c32])
    print(f"max relative error: {e:.3e} (fp64 coefficients), {e32:.3e} (fp32 coefficients)")
