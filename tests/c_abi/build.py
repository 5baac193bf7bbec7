"""Compile tests/c_abi/step_from_c.c against include/liteattn.h and libliteattn.so (gcc)."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
PKG = os.path.join(ROOT, "temporal_block_sparse_sm_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def build(out_dir: str) -> str:
    exe = os.path.join(out_dir, "step_from_c")
    cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(HERE, "step_from_c.c"), "-o", exe,
           "-L", PKG, "-lliteattn", "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm",
           "-Wl,-rpath," + PKG, "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe
