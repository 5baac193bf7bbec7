"""The C ABI used from plain C: tests/c_abi/step_from_c.c includes only
include/liteattn.h (and the CUDA runtime header for device memory) and links
libliteattn.so.  On CPU it checks argument validation and error strings; on a
GPU it runs one step whose output and mask are compared with the oracle."""
from __future__ import annotations

import math
import os
import subprocess

import numpy as np
import pytest

import oracle
from temporal_block_sparse_sm_b200 import build as lib_build
from tests.c_abi import build as c_build
from tests.helpers import bits_to_f64, random_qkv
from tests.parity import check_step


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    lib_build.build()
    return c_build.build(str(tmp_path_factory.mktemp("c_abi")))


def test_argument_checks_from_c(exe):
    res = subprocess.run([exe, "checks"], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0, res.stderr


@pytest.mark.gpu
def test_one_step_from_c_matches_oracle(exe, tmp_path):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, H, N, d = 1, 2, 1000, 64
    tau = math.log(1e-2)
    q, k, v = random_qkv(B, H, N, d, seed=5, scale_qk=2.0)  # bf16 bit patterns, as the other parity tests
    inp, out, msk = tmp_path / "in.bin", tmp_path / "out.bin", tmp_path / "mask.bin"
    np.concatenate([q.ravel(), k.ravel(), v.ravel()]).tofile(inp)
    res = subprocess.run([exe, "run", str(inp), str(out), str(msk)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    o = bits_to_f64(np.fromfile(out, dtype=np.uint16).reshape(B, H, N, d))
    Tq, Tk, W = oracle.tiles(N, d, d)
    mask = np.fromfile(msk, dtype=np.uint32).reshape(B * H * Tq, W)
    items = np.arange(B * H * Tq)
    full = np.full((B * H * Tq, W), 0xFFFFFFFF, dtype=np.uint32)
    full[:, W - 1] = (1 << (Tk % 32)) - 1 if Tk % 32 else 0xFFFFFFFF
    # the shared acceptance rule: masks within the margin, the oracle re-run with the
    # GPU's decision forced where a near-threshold tile flipped, absolute output bounds
    res = check_step(None, None, None, o, full, mask, B=B, H=H, N=N, d=d, Br=d, Bc=d, tau=tau, items=items,
                     host_qkv=(q, k, v))
    print(res)
