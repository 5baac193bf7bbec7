"""ctypes binding of the LiteAttention C ABI (include/liteattn.h).

Argument marshalling only: every step of the path runs in the CUDA library.
The ``lite_attn_*`` functions mirror the C entry points one to one (handles
are plain integers; errors raise :class:`LiteAttnError`).  :class:`Plan` and
:class:`Mask` wrap them for use with PyTorch tensors, which serve only as
device memory and streams.

There is no fallback: if ``libliteattn.so`` is missing or fails to load, the
first call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libliteattn.so")

LITE_OK = 0
LITE_ERR_INVALID_ARG = -1
LITE_ERR_UNSUPPORTED = -2
LITE_ERR_PLAN_MISMATCH = -3
LITE_ERR_ALLOC = -4
LITE_ERR_CUDA = -5
LITE_ERR_DEVICE_TIMEOUT = -6
LITE_ERR_DEVICE_CHECK = -7

LITE_LAYOUT_BHND = 0   # q, k, v, o as [B][H][N][d]
LITE_LAYOUT_BNHD = 1   # q, k, v, o as [B][N][H][d]
LITE_PRED_THRESHOLD = 0   # QK-Skip against a per-step threshold
LITE_PRED_RECALL = 1      # fixed recall p per step
_LAYOUTS = {"bhnd": LITE_LAYOUT_BHND, "bnhd": LITE_LAYOUT_BNHD}


class LiteAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {error_string(code)} ({code})")


class Stats(ctypes.Structure):
    _fields_ = [
        ("tiles_total", ctypes.c_int64), ("live_in", ctypes.c_int64), ("qk_tiles", ctypes.c_int64),
        ("pv_tiles", ctypes.c_int64), ("newly_dead", ctypes.c_int64), ("live_out", ctypes.c_int64),
        ("skip_fraction", ctypes.c_double), ("executed_flops", ctypes.c_double), ("dense_flops", ctypes.c_double),
        ("cum_qk_tiles", ctypes.c_int64), ("cum_pv_tiles", ctypes.c_int64), ("cum_steps", ctypes.c_int64),
        ("device_status", ctypes.c_int32), ("last_step", ctypes.c_int32),
    ]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


_lib = None
_VP = ctypes.c_void_p
_I = ctypes.c_int

# name -> (restype, argtypes): the exported symbols of include/liteattn.h
SIGNATURES = {
    "lite_attn_plan_create": (_I, [ctypes.POINTER(_VP), _I, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_float), _I]),
    "lite_attn_plan_create_ex": (_I, [ctypes.POINTER(_VP), _I, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_float),
                                      _I, _I, _I]),
    "lite_attn_plan_create_varlen": (_I, [ctypes.POINTER(_VP), _I, _I, _VP, _I, _I, _I,
                                          ctypes.POINTER(ctypes.c_float), _I]),
    "lite_attn_plan_create_recall": (_I, [ctypes.POINTER(_VP), _I, _I, _I, _I, _I, _I,
                                          ctypes.POINTER(ctypes.c_float), _I, _I, _I]),
    "lite_attn_plan_predicate": (_I, [_VP, ctypes.POINTER(_I)]),
    "lite_attn_plan_create_opts": (_I, [ctypes.POINTER(_VP), _I, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_float),
                                        _I, _VP]),
    "lite_attn_plan_pair_tiles": (_I, [_VP, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "lite_attn_plan_destroy": (_I, [_VP]),
    "lite_attn_plan_info": (_I, [_VP, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I),
                                 ctypes.POINTER(_I)]),
    "lite_attn_mask_create": (_I, [_VP, ctypes.POINTER(_VP)]),
    "lite_attn_mask_destroy": (_I, [_VP]),
    "lite_attn_mask_reset": (_I, [_VP, _VP]),
    "lite_attn_mask_import": (_I, [_VP, _VP, _VP]),
    "lite_attn_mask_export": (_I, [_VP, _VP, _VP]),
    "lite_attn_mask_export_lists": (_I, [_VP, _VP, _VP, _VP, _VP]),
    "lite_attn_mask_compare": (_I, [_VP, _VP, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64), _VP]),
    "lite_attn_step": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _VP]),
    "lite_attn_output_error": (_I, [_VP, _VP, _VP, ctypes.POINTER(ctypes.c_double), _VP]),
    "lite_attn_stats": (_I, [_VP, _VP, ctypes.POINTER(Stats)]),
    "lite_attn_timing_enable": (_I, [_VP, _I]),
    "lite_attn_timing_read": (_I, [_VP, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double),
                                   ctypes.POINTER(ctypes.c_int64)]),
    "lite_attn_compact_noalloc": (_I, [_VP, _I, _I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP]),
    "lite_attn_launch_count": (ctypes.c_int64, []),
    "lite_attn_error_string": (ctypes.c_char_p, [_I]),
}


def load(path: str = LIB_PATH):
    """Load the CUDA library (raises if it is missing: there is no CPU path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"LiteAttention CUDA library not built ({path}); run __graft_entry__.build()")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(rc: int, where: str):
    if rc != LITE_OK:
        raise LiteAttnError(rc, where)


def error_string(code: int) -> str:
    try:
        return load().lite_attn_error_string(code).decode()
    except Exception:  # library missing: still give a readable message
        return str(code)


def _stream_ptr(stream) -> Optional[int]:
    """cudaStream_t handle: the current device's current stream for None."""
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ----------------------------------------------------------------- raw C-ABI mirrors
def lite_attn_plan_create(B: int, H: int, N: int, d: int, Br: int, Bc: int, threshold_schedule: Sequence[float]) -> int:
    taus = (ctypes.c_float * len(threshold_schedule))(*[float(t) for t in threshold_schedule])
    h = _VP()
    _check(load().lite_attn_plan_create(ctypes.byref(h), B, H, N, d, Br, Bc, taus, len(threshold_schedule)),
           "lite_attn_plan_create")
    return h.value


def lite_attn_plan_create_ex(B: int, H: int, N: int, d: int, Br: int, Bc: int, threshold_schedule: Sequence[float],
                             layout: int, heads_total: int = 0) -> int:
    taus = (ctypes.c_float * len(threshold_schedule))(*[float(t) for t in threshold_schedule])
    h = _VP()
    _check(load().lite_attn_plan_create_ex(ctypes.byref(h), B, H, N, d, Br, Bc, taus, len(threshold_schedule),
                                           layout, heads_total), "lite_attn_plan_create_ex")
    return h.value


def lite_attn_plan_create_varlen(seq_lens: Sequence[int], H: int, d: int, Br: int, Bc: int,
                                 threshold_schedule: Sequence[float]) -> int:
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    taus = (ctypes.c_float * len(threshold_schedule))(*[float(t) for t in threshold_schedule])
    h = _VP()
    _check(load().lite_attn_plan_create_varlen(ctypes.byref(h), len(lens), H, lens.ctypes.data, d, Br, Bc, taus,
                                               len(threshold_schedule)), "lite_attn_plan_create_varlen")
    return h.value


def lite_attn_plan_create_recall(B: int, H: int, N: int, d: int, Br: int, Bc: int, recall_schedule: Sequence[float],
                                 layout: int = 0, heads_total: int = 0) -> int:
    ps = (ctypes.c_float * len(recall_schedule))(*[float(x) for x in recall_schedule])
    h = _VP()
    _check(load().lite_attn_plan_create_recall(ctypes.byref(h), B, H, N, d, Br, Bc, ps, len(recall_schedule),
                                               layout, heads_total), "lite_attn_plan_create_recall")
    return h.value


class PlanOptions(ctypes.Structure):
    """lite_attn_plan_options_t."""
    _fields_ = [("layout", ctypes.c_int), ("heads_total", ctypes.c_int), ("predicate", ctypes.c_int),
                ("pair_stride", ctypes.c_int)]


def lite_attn_plan_create_opts(B: int, H: int, N: int, d: int, Br: int, Bc: int, schedule: Sequence[float],
                               layout: int = 0, heads_total: int = 0, predicate: int = 0, pair_stride: int = 0) -> int:
    arr = (ctypes.c_float * len(schedule))(*[float(x) for x in schedule])
    opts = PlanOptions(layout, heads_total, predicate, pair_stride)
    h = _VP()
    _check(load().lite_attn_plan_create_opts(ctypes.byref(h), B, H, N, d, Br, Bc, arr, len(schedule),
                                             ctypes.byref(opts)), "lite_attn_plan_create_opts")
    return h.value


def lite_attn_plan_pair_tiles(plan: int, pair: int):
    a, b = _I(), _I()
    _check(load().lite_attn_plan_pair_tiles(plan, pair, ctypes.byref(a), ctypes.byref(b)),
           "lite_attn_plan_pair_tiles")
    return a.value, b.value


def lite_attn_plan_predicate(plan: int) -> int:
    x = _I()
    _check(load().lite_attn_plan_predicate(plan, ctypes.byref(x)), "lite_attn_plan_predicate")
    return x.value


def lite_attn_plan_destroy(plan: int):
    _check(load().lite_attn_plan_destroy(plan), "lite_attn_plan_destroy")


def lite_attn_plan_info(plan: int):
    a, b, c, d = _I(), _I(), _I(), _I()
    _check(load().lite_attn_plan_info(plan, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c), ctypes.byref(d)),
           "lite_attn_plan_info")
    return {"Tq": a.value, "Tk": b.value, "W": c.value, "G": d.value}


def lite_attn_mask_create(plan: int) -> int:
    h = _VP()
    _check(load().lite_attn_mask_create(plan, ctypes.byref(h)), "lite_attn_mask_create")
    return h.value


def lite_attn_mask_destroy(mask: int):
    _check(load().lite_attn_mask_destroy(mask), "lite_attn_mask_destroy")


def lite_attn_mask_reset(mask: int, stream=None):
    _check(load().lite_attn_mask_reset(mask, _stream_ptr(stream)), "lite_attn_mask_reset")


def lite_attn_mask_import(mask: int, host_bits: np.ndarray, stream=None):
    arr = np.ascontiguousarray(host_bits, dtype=np.uint32)
    _check(load().lite_attn_mask_import(mask, arr.ctypes.data, _stream_ptr(stream)), "lite_attn_mask_import")


def lite_attn_mask_export(mask: int, rows: int, W: int, stream=None) -> np.ndarray:
    out = np.zeros((rows, W), dtype=np.uint32)
    _check(load().lite_attn_mask_export(mask, out.ctypes.data, _stream_ptr(stream)), "lite_attn_mask_export")
    return out


def lite_attn_mask_export_lists(mask: int, G: int, Tk: int, stream=None):
    lst = np.zeros((G, Tk), dtype=np.uint32)
    cnt = np.zeros(G, dtype=np.int32)
    order = np.zeros(G, dtype=np.int32)
    _check(load().lite_attn_mask_export_lists(mask, lst.ctypes.data, cnt.ctypes.data, order.ctypes.data,
                                              _stream_ptr(stream)), "lite_attn_mask_export_lists")
    return lst, cnt, order


def lite_attn_mask_compare(a: int, b: int, stream=None):
    """(tiles live in a and not in b, tiles live in b and not in a)."""
    x, y = ctypes.c_int64(), ctypes.c_int64()
    _check(load().lite_attn_mask_compare(a, b, ctypes.byref(x), ctypes.byref(y), _stream_ptr(stream)),
           "lite_attn_mask_compare")
    return x.value, y.value


def lite_attn_step(plan: int, q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, mask_in: int, mask_out: int,
                   step: int, stream=None):
    _check(load().lite_attn_step(plan, q_ptr, k_ptr, v_ptr, o_ptr, mask_in, mask_out, step, _stream_ptr(stream)),
           "lite_attn_step")


def lite_attn_output_error(plan: int, o_ptr: int, ref_ptr: int, stream=None):
    """(sum |o - o_ref|, max |o - o_ref|, sum |o_ref|) over the plan's B*H*N*d elements."""
    out = (ctypes.c_double * 3)()
    _check(load().lite_attn_output_error(plan, o_ptr, ref_ptr, out, _stream_ptr(stream)), "lite_attn_output_error")
    return out[0], out[1], out[2]


def lite_attn_stats(plan: int, mask: int, check: bool = True) -> dict:
    s = Stats()
    rc = load().lite_attn_stats(plan, mask, ctypes.byref(s))
    if check:
        _check(rc, "lite_attn_stats")
    d = s.as_dict()
    d["rc"] = rc
    return d


def lite_attn_timing_enable(plan: int, enable: bool = True):
    _check(load().lite_attn_timing_enable(plan, 1 if enable else 0), "lite_attn_timing_enable")


def lite_attn_timing_read(plan: int):
    a, s, n = ctypes.c_double(), ctypes.c_double(), ctypes.c_int64()
    _check(load().lite_attn_timing_read(plan, ctypes.byref(a), ctypes.byref(s), ctypes.byref(n)),
           "lite_attn_timing_read")
    return a.value, s.value, n.value


def lite_attn_compact_noalloc(bits_ptr: int, B: int, H: int, N: int, Br: int, Bc: int, list_ptr: int, cnt_ptr: int,
                              order_ptr: int, live_total_ptr: int, stream=None):
    """Compaction into caller-owned device buffers; the library allocates nothing."""
    _check(load().lite_attn_compact_noalloc(bits_ptr, B, H, N, Br, Bc, list_ptr, cnt_ptr, order_ptr, live_total_ptr,
                                            _stream_ptr(stream)), "lite_attn_compact_noalloc")


def lite_attn_launch_count() -> int:
    return int(load().lite_attn_launch_count())


def lite_attn_error_string(code: int) -> str:
    return load().lite_attn_error_string(code).decode()


# ----------------------------------------------------------------- object layer
def _current_device() -> Optional[int]:
    """The calling thread's current CUDA device (None without CUDA: plan creation then
    fails in the library with its own error code)."""
    import torch
    return torch.cuda.current_device() if torch.cuda.is_available() else None


class Plan:
    """A LiteAttention plan: fixed (B, H, N, d, Br, Bc), a T-step threshold schedule and
    the tensor layout ("bhnd": [B, H, N, d], the default; "bnhd": [B, N, H, d]).

    With ``heads_total`` the plan covers heads [head_offset, head_offset + H) of
    tensors that hold ``heads_total`` heads (one shard of the heads, e.g. per GPU);
    ``step`` then takes the full tensors.

    With ``seq_lens`` the plan covers B = len(seq_lens) sequences of those lengths
    packed token-major: tensors of shape [sum(seq_lens), H, d] (B and N are then
    taken from seq_lens; pass None for them).

    ``predicate`` is "threshold" (QK-Skip; ``taus`` are the per-step thresholds)
    or "recall" (the fixed-recall predicate; ``taus`` are then the per-step recall
    targets p in (0, 1]).

    ``pair_stride`` chooses which query tiles share a work item (1: adjacent; s > 1:
    tile i with tile i + s in blocks of 2s, e.g. s = tiles per video frame); results
    do not depend on it."""

    def __init__(self, B: Optional[int], H: int, N: Optional[int], d: int, Br: int, Bc: int, taus: Sequence[float],
                 layout: str = "bhnd", heads_total: Optional[int] = None, head_offset: int = 0,
                 seq_lens: Optional[Sequence[int]] = None, predicate: str = "threshold", pair_stride: int = 1):
        if predicate not in ("threshold", "recall"):
            raise ValueError("predicate must be 'threshold' or 'recall'")
        self.predicate = predicate
        self.pair_stride = int(pair_stride)
        if self.pair_stride != 1 and seq_lens is not None:
            raise ValueError("a pair stride needs a fixed-length plan")
        if predicate == "recall" and seq_lens is not None:
            raise ValueError("fixed-recall plans are fixed-length")
        if seq_lens is not None:
            lens = [int(x) for x in seq_lens]
            if not lens or min(lens) < 1:
                raise ValueError("seq_lens must be positive lengths")
            if (B is not None and B != len(lens)) or (N is not None and N != max(lens)):
                raise ValueError("B and N of a variable-length plan come from seq_lens")
            if heads_total not in (None, H) or head_offset:
                raise ValueError("variable-length plans cover all heads")
            self.B, self.H, self.N, self.d, self.Br, self.Bc = len(lens), H, max(lens), d, Br, Bc
            self.layout, self.heads_total, self.head_offset, self.seq_lens = "varlen", H, 0, lens
            self.taus = [float(t) for t in taus]
            self.device = _current_device()
            self.handle = lite_attn_plan_create_varlen(lens, H, d, Br, Bc, self.taus)
            info = lite_attn_plan_info(self.handle)
            self.Tq, self.Tk, self.W, self.G = info["Tq"], info["Tk"], info["W"], info["G"]
            self.R = self.B * H * self.Tq
            return
        self.seq_lens = None
        if layout not in _LAYOUTS:
            raise ValueError(f"layout must be one of {sorted(_LAYOUTS)}")
        Ht = H if heads_total is None else int(heads_total)
        if not (0 <= head_offset and head_offset + H <= Ht):
            raise ValueError("the head range must lie inside the tensors' heads")
        self.B, self.H, self.N, self.d, self.Br, self.Bc = B, H, N, d, Br, Bc
        self.layout, self.heads_total, self.head_offset = layout, Ht, head_offset
        self.taus = [float(t) for t in taus]
        self.device = _current_device()
        if self.pair_stride != 1:
            self.handle = lite_attn_plan_create_opts(B, H, N, d, Br, Bc, self.taus, _LAYOUTS[layout], Ht,
                                                     LITE_PRED_RECALL if predicate == "recall" else LITE_PRED_THRESHOLD,
                                                     self.pair_stride)
        elif predicate == "recall":
            self.handle = lite_attn_plan_create_recall(B, H, N, d, Br, Bc, self.taus, _LAYOUTS[layout], Ht)
        elif layout == "bhnd" and Ht == H:
            self.handle = lite_attn_plan_create(B, H, N, d, Br, Bc, self.taus)
        else:
            self.handle = lite_attn_plan_create_ex(B, H, N, d, Br, Bc, self.taus, _LAYOUTS[layout], Ht)
        info = lite_attn_plan_info(self.handle)
        self.Tq, self.Tk, self.W, self.G = info["Tq"], info["Tk"], info["W"], info["G"]
        self.R = B * H * self.Tq

    def mask(self) -> "Mask":
        return Mask(self)

    def stream(self, stream=None):
        """The stream a call runs on: `stream`, else the current stream of the plan's device
        (the plan's device may differ from the thread's current device)."""
        if stream is not None:
            return stream
        import torch
        return torch.cuda.current_stream(self.device)

    @property
    def shape(self):
        """Shape of q, k, v and o for this plan's layout (all heads of the tensors)."""
        if self.seq_lens is not None:
            return (sum(self.seq_lens), self.H, self.d)
        if self.layout == "bnhd":
            return (self.B, self.N, self.heads_total, self.d)
        return (self.B, self.heads_total, self.N, self.d)

    def _ptr(self, t) -> int:
        """Address of the plan's first head in tensor t."""
        per_head = self.d if self.layout in ("bnhd", "varlen") else self.N * self.d
        return t.data_ptr() + 2 * self.head_offset * per_head

    def _check_tensor(self, t, name):
        import torch
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
                and tuple(t.shape) == self.shape):
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {self.shape}")

    def step(self, q, k, v, o, mask_in: "Mask", mask_out: "Mask", step: int, stream=None):
        for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
            self._check_tensor(t, nm)
        lite_attn_step(self.handle, self._ptr(q), self._ptr(k), self._ptr(v), self._ptr(o), mask_in.handle,
                       mask_out.handle, step, self.stream(stream))

    def stats(self, mask: "Mask", check: bool = True) -> dict:
        return lite_attn_stats(self.handle, mask.handle, check)

    def output_error(self, o, o_ref, stream=None) -> dict:
        """Error of o against o_ref: relative L1 (sum |o - o_ref| / sum |o_ref|) and max-abs."""
        self._check_tensor(o, "o")
        self._check_tensor(o_ref, "o_ref")
        sd, mx, sr = lite_attn_output_error(self.handle, o.data_ptr(), o_ref.data_ptr(), self.stream(stream))
        return {"rel_l1": sd / sr if sr > 0 else (0.0 if sd == 0 else math.inf), "max_abs": mx,
                "sum_abs_diff": sd, "sum_abs_ref": sr}

    def timing(self, enable: bool = True):
        lite_attn_timing_enable(self.handle, enable)

    def timing_read(self):
        return lite_attn_timing_read(self.handle)

    def close(self):
        if getattr(self, "handle", None):
            lite_attn_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Mask:
    """A persistent skip mask of a plan (created all-live)."""

    def __init__(self, plan: Plan):
        self.plan = plan
        self.handle = lite_attn_mask_create(plan.handle)

    def reset(self, stream=None):
        lite_attn_mask_reset(self.handle, self.plan.stream(stream))

    def import_bits(self, bits: np.ndarray, stream=None):
        bits = np.asarray(bits, dtype=np.uint32).reshape(self.plan.R, self.plan.W)
        lite_attn_mask_import(self.handle, bits, self.plan.stream(stream))

    def export_bits(self, stream=None) -> np.ndarray:
        return lite_attn_mask_export(self.handle, self.plan.R, self.plan.W, self.plan.stream(stream))

    def export_lists(self, stream=None):
        return lite_attn_mask_export_lists(self.handle, self.plan.G, self.plan.Tk, self.plan.stream(stream))

    def compare(self, other: "Mask", stream=None):
        """(tiles live here and dead in `other`, tiles live in `other` and dead here)."""
        return lite_attn_mask_compare(self.handle, other.handle, self.plan.stream(stream))

    def close(self):
        if getattr(self, "handle", None):
            lite_attn_mask_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def schedule_loglinear(T: int, lo: float = 1e-6, hi: float = 1e-3):
    """Thresholds rising linearly in the log domain from ln(lo) to ln(hi) over T steps."""
    a, b = math.log(lo), math.log(hi)
    return [a + (b - a) * t / (T - 1) if T > 1 else a for t in range(T)]
