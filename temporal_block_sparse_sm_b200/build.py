"""Build the in-tree CUDA library ``libliteattn.so`` for sm_100a with nvcc."""
from __future__ import annotations

import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libliteattn.so")
PROF_LIB = os.path.join(PKG, "libliteattn_prof.so")   # cycle-counter build, for kernel analysis only
DEBUG_LIB = os.path.join(PKG, "libliteattn_debug.so")  # device-side checks of every work item (LITE_DEBUG_CHECKS)


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, profile: bool = False, debug: bool = False) -> str:
    """Compile csrc/liteattn.cu (and the headers it includes) into libliteattn.so.

    profile=True builds libliteattn_prof.so with per-CTA cycle counters instead;
    debug=True builds libliteattn_debug.so, whose attention kernel checks every
    work item (order, count, list entries) before using it and reports a bad one
    as LITE_ERR_DEVICE_CHECK."""
    out = PROF_LIB if profile else DEBUG_LIB if debug else LIB
    if not force and not profile and not needs_build(out):
        return out
    tmp = out + f".tmp{os.getpid()}"
    flags = (["-DLITE_PROFILE"] if profile else []) + (["-DLITE_DEBUG_CHECKS"] if debug else [])
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC,
           "-Xptxas", "-v" if verbose else "-O3"] + flags + [os.path.join(CSRC, "liteattn.cu"), "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stdout + res.stderr)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose="-v" in sys.argv))
