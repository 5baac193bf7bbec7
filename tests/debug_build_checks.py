"""Steps run with the checked build (libliteattn_debug.so), in a process of its own.

First the softmax's two exponential paths are held against exact 2^x on the
device (the checked build exports them as lite_attn_debug_exp2).

The checked build's attention kernel validates every work item (the order
entry, the count, each live-list entry) before using it and records a bad one
as LITE_ERR_DEVICE_CHECK.  This script runs config 1 (every step, parity with
the oracle), partial-tile edge shapes, random imported masks (5-80% live) and
an all-dead mask through it; every step must leave the status word at OK.
Run by tests/test_gpu_debug_build.py (the binding loads one library per process).
"""
from __future__ import annotations

import math
import sys

import numpy as np
import torch


def check_exp2_paths(lib) -> None:
    """The softmax's two exponential paths, run on the device through the checked
    build's lite_attn_debug_exp2, against exact 2^x (fp64).  On [-125, 0] the FMA-pipe
    polynomial stays within its fitted relative-error bound (7.5e-5, plus fp32
    evaluation), and MUFU ex2 within 2^-20.  Below -125 (to -inf) the polynomial gives
    finite values in [0, 2^-125]."""
    import ctypes

    fn = lib.lite_attn_debug_exp2
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64]
    grid = np.linspace(-125.0, 0.0, 1 << 20).astype(np.float32)
    extra = np.array([0.0, -0.0, -1e-7, -0.5, -0.49999997, -0.50000006, -1.5, -124.5, -125.0, -125.5, -126.0,
                      -130.0, -1000.0, -np.inf], dtype=np.float32)
    x = np.concatenate([grid, extra])
    xd = torch.from_numpy(x).cuda()
    yp, ym = torch.empty_like(xd), torch.empty_like(xd)
    assert fn(xd.data_ptr(), yp.data_ptr(), ym.data_ptr(), x.size) == 0
    yp, ym = yp.cpu().numpy().astype(np.float64), ym.cpu().numpy().astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    inr = x >= -125.0
    rel_p = float(np.abs(yp[inr] / exact[inr] - 1.0).max())
    rel_m = float(np.abs(ym[inr] / exact[inr] - 1.0).max())
    assert rel_p <= 7.6e-5, rel_p
    assert rel_m <= 2.0 ** -20, rel_m
    low = yp[~inr]
    assert np.all(np.isfinite(low)) and np.all(low >= 0.0) and np.all(low <= 2.0 ** -125), low
    print(f"exp2 paths: polynomial max relative error {rel_p:.3e}, MUFU ex2 {rel_m:.3e}")


def main() -> int:
    from temporal_block_sparse_sm_b200 import build, liteattn, synthetic
    from tests.parity import check_step

    lib = liteattn.load(build.build(debug=True))
    check_exp2_paths(lib)
    cfg = synthetic.CONFIGS["c1"]
    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, cfg.taus())
    mask = plan.mask()
    wl = synthetic.Workload(cfg, seed=0, device="cuda")
    o = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
    for t in range(cfg.T):
        q, k, v = wl.inputs(t)
        bits_in = mask.export_bits()
        plan.step(q, k, v, o, mask, mask, t)
        check_step(q, k, v, o, bits_in, mask.export_bits(), B=cfg.B, H=cfg.H, N=cfg.N, d=cfg.d, Br=cfg.Br,
                   Bc=cfg.Bc, tau=plan.taus[t], items=np.arange(plan.R), step=t)
        assert plan.stats(mask)["device_status"] == 0
    g = torch.Generator(device="cuda").manual_seed(9)
    for d, N in ((64, 1), (64, 65), (64, 200), (128, 129), (128, 1000), (64, 70000)):
        p = liteattn.Plan(2, 3, N, d, d, d, [math.log(1e-2), -math.inf])
        m = p.mask()
        q, k, v = (torch.randn(2, 3, N, d, generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
        o = torch.empty_like(q)
        p.step(q, k, v, o, m, m, 0)
        for frac in (0.05, 0.3, 0.8, 0.0):
            m.import_bits(synthetic.random_live_bits(p.R, p.Tk, frac, seed=int(100 * frac), keep_first=frac > 0)
                          .numpy().astype(np.uint32))
            p.step(q, k, v, o, m, m, 1)
        st = p.stats(m)
        assert st["device_status"] == 0, (d, N, st)
    print("checked build: all work items valid")
    return 0


if __name__ == "__main__":
    sys.exit(main())
