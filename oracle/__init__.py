"""CPU oracle for one LiteAttention denoising step -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or runs anything here, and this
package never imports the product.

The arithmetic lives in plain fp64 C (OpenMP over work items); this module
only compiles it with gcc and marshals numpy arrays:
  * ``lite_oracle.c`` -- the LiteAttention step with the QK-Skip threshold test
    ("LiteAttention: Temporal Sparse Attention for Diffusion Transformers",
    skill page: "Core Concept", "Architecture Overview"; the LiteAttention
    abstract);
  * ``recall_oracle.c`` -- the same step with the fixed-recall ("cumulative
    energy") skip predicate ("Training-free sparse attention based on
    cumulative energy filtering", abstract).
What each computes, and the reading of its page, is documented at its top.

Pins: ``step`` is pinned by ``tests/test_oracle_pins.py`` against library
softmax attention, a closed-form prefix-max decision rule, a subset
fixed-point characterisation, the analytic skipped-mass error bound and the
hand-built fixtures in ``tests/golden/``; ``step_recall`` by
``tests/test_oracle_recall.py`` against library attention at p = 1 and on the
kept keys, the recall floor measured from library softmax probabilities, and
closed-form decisions on tiles of constant logits.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = [os.path.join(_HERE, "lite_oracle.c"), os.path.join(_HERE, "recall_oracle.c")]
_LIB = os.path.join(_HERE, "liblite_oracle.so")
_lib = None


def compile_library(sources, out: str) -> str:
    """gcc -O2 -fopenmp the given C files into one shared library."""
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", *sources, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc, -O2, OpenMP).  Returns its path."""
    if force or not os.path.exists(_LIB) or any(os.path.getmtime(_LIB) < os.path.getmtime(s) for s in SOURCES):
        tmp = _LIB + f".tmp{os.getpid()}"
        compile_library(SOURCES, tmp)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    """Load the oracle library.  LITE_ORACLE_LIB, when set, names another build of
    the oracle sources to load instead: the mutation tests set it to run the pins
    against copies with a planted mistake.  Normal use never sets it."""
    global _lib
    if _lib is None:
        path = os.environ.get("LITE_ORACLE_LIB")
        if not path:
            build()
            path = _LIB
        lib = ctypes.CDLL(path)
        lib.lo_step.restype = ctypes.c_int
        lib.lo_step.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int64,
            ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ]
        lib.lo_step_recall.restype = ctypes.c_int
        lib.lo_step_recall.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int64,
            ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ]
        lib.lo_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().lo_max_threads())


def tiles(N: int, Br: int, Bc: int):
    """(Tq, Tk, W): query tiles, key tiles, 32-bit words per mask row."""
    Tq = -(-N // Br)
    Tk = -(-N // Bc)
    return Tq, Tk, -(-Tk // 32)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def step(q: np.ndarray, k: np.ndarray, v: np.ndarray, *, B: int, H: int, N: int, d: int,
         Br: int, Bc: int, tau: float, items, mask_in: np.ndarray,
         force: Optional[np.ndarray] = None, threads: int = 0) -> dict:
    """Run the oracle step on the given work items.

    q, k, v: uint16 arrays holding bf16 bit patterns, shape [B, H, N, d].
    items: work-item ids (b*H + h)*Tq + i.
    mask_in: uint32 [n_items, W] -- each item's mask_in row (teacher forcing).
    force: optional int8 [n_items, Tk] (-1 own decision, 0 dead, 1 live).
    Returns dict with o [n,Br,d] f64, mask_out [n,W] u32, D [n,Tk] f64,
    m_fin [n,Br], l_fin [n,Br].
    """
    lib = _load()
    Tq, Tk, W = tiles(N, Br, Bc)
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    for a in (q, k, v):
        if a.size != B * H * N * d:
            raise ValueError("q/k/v must hold B*H*N*d elements")
    items = np.ascontiguousarray(np.asarray(items, dtype=np.int64).reshape(-1))
    n = items.shape[0]
    mask_in = np.ascontiguousarray(mask_in, dtype=np.uint32).reshape(n, W)
    if force is not None:
        force = np.ascontiguousarray(force, dtype=np.int8).reshape(n, Tk)
    o = np.zeros((n, Br, d), dtype=np.float64)
    mask_out = np.zeros((n, W), dtype=np.uint32)
    D = np.full((n, Tk), np.nan, dtype=np.float64)
    m_fin = np.full((n, Br), np.nan, dtype=np.float64)
    l_fin = np.full((n, Br), np.nan, dtype=np.float64)
    rc = lib.lo_step(B, H, N, d, Br, Bc, float(tau), _ptr(q), _ptr(k), _ptr(v),
                     _ptr(items), n, _ptr(mask_in), _ptr(force),
                     _ptr(o), _ptr(mask_out), _ptr(D), _ptr(m_fin), _ptr(l_fin), int(threads))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return {"o": o, "mask_out": mask_out, "D": D, "m_fin": m_fin, "l_fin": l_fin}


def step_recall(q: np.ndarray, k: np.ndarray, v: np.ndarray, *, B: int, H: int, N: int, d: int,
                Br: int, Bc: int, p: float, items, mask_in: np.ndarray,
                force: Optional[np.ndarray] = None, threads: int = 0) -> dict:
    """Run the fixed-recall oracle step (recall target 0 < p <= 1) on the given work items.

    Arguments as :func:`step`.  Returns dict with o [n,Br,d] f64, mask_out [n,W] u32,
    E [n,Tk] f64 (decision statistic: the tile is skipped iff E <= 0; NaN where not
    tested), m_fin, l_fin, z_fin [n,Br] (final running max, kept mass and skipped-mass
    bound of each row).
    """
    lib = _load()
    Tq, Tk, W = tiles(N, Br, Bc)
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    for a in (q, k, v):
        if a.size != B * H * N * d:
            raise ValueError("q/k/v must hold B*H*N*d elements")
    items = np.ascontiguousarray(np.asarray(items, dtype=np.int64).reshape(-1))
    n = items.shape[0]
    mask_in = np.ascontiguousarray(mask_in, dtype=np.uint32).reshape(n, W)
    if force is not None:
        force = np.ascontiguousarray(force, dtype=np.int8).reshape(n, Tk)
    o = np.zeros((n, Br, d), dtype=np.float64)
    mask_out = np.zeros((n, W), dtype=np.uint32)
    E = np.full((n, Tk), np.nan, dtype=np.float64)
    m_fin = np.full((n, Br), np.nan, dtype=np.float64)
    l_fin = np.full((n, Br), np.nan, dtype=np.float64)
    z_fin = np.full((n, Br), np.nan, dtype=np.float64)
    rc = lib.lo_step_recall(B, H, N, d, Br, Bc, float(p), _ptr(q), _ptr(k), _ptr(v),
                            _ptr(items), n, _ptr(mask_in), _ptr(force),
                            _ptr(o), _ptr(mask_out), _ptr(E), _ptr(m_fin), _ptr(l_fin), _ptr(z_fin), int(threads))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return {"o": o, "mask_out": mask_out, "E": E, "m_fin": m_fin, "l_fin": l_fin, "z_fin": z_fin}


def all_live_rows(n_items: int, N: int, Bc: int) -> np.ndarray:
    """mask_in rows with every key tile live (bits >= Tk stay 0)."""
    Tk = -(-N // Bc)
    W = -(-Tk // 32)
    rows = np.zeros((n_items, W), dtype=np.uint32)
    for j in range(Tk):
        rows[:, j >> 5] |= np.uint32(1 << (j & 31))
    return rows


def bits_to_bool(rows: np.ndarray, Tk: int) -> np.ndarray:
    """[n, W] uint32 -> [n, Tk] bool."""
    rows = np.asarray(rows, dtype=np.uint32)
    j = np.arange(Tk)
    return ((rows[:, j >> 5] >> (j & 31).astype(np.uint32)) & 1).astype(bool)


def bool_to_bits(live: np.ndarray) -> np.ndarray:
    """[n, Tk] bool -> [n, W] uint32."""
    live = np.asarray(live, dtype=bool)
    n, Tk = live.shape
    W = -(-Tk // 32)
    rows = np.zeros((n, W), dtype=np.uint32)
    for j in range(Tk):
        rows[:, j >> 5] |= live[:, j].astype(np.uint32) << np.uint32(j & 31)
    return rows


NEG_INF = -math.inf
