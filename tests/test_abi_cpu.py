"""C-ABI checks that need no GPU: the library builds, loads and exports every
symbol include/liteattn.h declares; host-side argument checks and host fault
injection return the documented codes without touching a device."""
from __future__ import annotations

import ctypes
import math
import os
import re
import subprocess

import pytest

from temporal_block_sparse_sm_b200 import build as lib_build
from temporal_block_sparse_sm_b200 import liteattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names.update(re.findall(r"\b(lite_attn_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    lib_build.build()
    return liteattn.load()


def test_library_exports_every_declared_symbol(lib):
    declared = header_functions()
    assert declared, "no declarations found"
    out = subprocess.run(["nm", "-D", "--defined-only", liteattn.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\b(lite_attn_\w+)\b", out))
    assert declared <= exported, declared - exported
    for name in declared:
        assert hasattr(lib, name)


def test_debug_build_exports_the_same_symbols():
    path = lib_build.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    declared = header_functions()
    assert declared <= set(re.findall(r"\b(lite_attn_\w+)\b", out))


def test_binding_covers_header_exactly():
    assert set(liteattn.SIGNATURES) == header_functions()


def test_error_strings(lib):
    for code in range(0, -7, -1):
        s = liteattn.lite_attn_error_string(code)
        assert s and s != "unknown error"
    assert liteattn.lite_attn_error_string(-99) == "unknown error"


def _create(B=1, H=1, N=128, d=64, Br=64, Bc=64, taus=(-1.0,)):
    lib = liteattn.load()
    arr = (ctypes.c_float * len(taus))(*taus)
    h = ctypes.c_void_p()
    rc = lib.lite_attn_plan_create(ctypes.byref(h), B, H, N, d, Br, Bc, arr, len(taus))
    return rc, h


@pytest.mark.parametrize("kw,code", [
    (dict(taus=(0.5,)), liteattn.LITE_ERR_INVALID_ARG),
    (dict(taus=(float("nan"),)), liteattn.LITE_ERR_INVALID_ARG),
    (dict(B=0), liteattn.LITE_ERR_INVALID_ARG),
    (dict(H=0), liteattn.LITE_ERR_INVALID_ARG),
    (dict(N=0), liteattn.LITE_ERR_UNSUPPORTED),
    (dict(N=(1 << 20) + 1), liteattn.LITE_ERR_UNSUPPORTED),
    (dict(d=128, Br=64, Bc=64), liteattn.LITE_ERR_UNSUPPORTED),
    (dict(d=64, Br=128, Bc=64), liteattn.LITE_ERR_UNSUPPORTED),
    (dict(d=96, Br=128, Bc=128), liteattn.LITE_ERR_UNSUPPORTED),
])
def test_plan_argument_checks(lib, kw, code):
    rc, h = _create(**kw)
    assert rc == code
    assert not h.value


def test_plan_null_out_and_empty_schedule(lib):
    arr = (ctypes.c_float * 1)(-1.0)
    assert lib.lite_attn_plan_create(None, 1, 1, 64, 64, 64, 64, arr, 1) == liteattn.LITE_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert lib.lite_attn_plan_create(ctypes.byref(h), 1, 1, 64, 64, 64, 64, None, 1) == liteattn.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_plan_create(ctypes.byref(h), 1, 1, 64, 64, 64, 64, arr, 0) == liteattn.LITE_ERR_INVALID_ARG


@pytest.mark.parametrize("layout", [-1, 2, 7])
def test_plan_rejects_unknown_layout(lib, layout):
    arr = (ctypes.c_float * 1)(-1.0)
    h = ctypes.c_void_p()
    assert lib.lite_attn_plan_create_ex(ctypes.byref(h), 1, 1, 64, 64, 64, 64, arr, 1, layout, 0) == \
        liteattn.LITE_ERR_INVALID_ARG
    assert not h.value


@pytest.mark.parametrize("layout", [liteattn.LITE_LAYOUT_BHND, liteattn.LITE_LAYOUT_BNHD])
def test_plan_layouts_pass_validation(lib, monkeypatch, layout):
    # both layouts get past argument checks; the injected allocation fault proves it
    monkeypatch.setenv("LITE_ATTN_FAULT", "alloc")
    arr = (ctypes.c_float * 1)(-1.0)
    h = ctypes.c_void_p()
    assert lib.lite_attn_plan_create_ex(ctypes.byref(h), 2, 3, 1000, 128, 128, 128, arr, 1, layout, 0) == \
        liteattn.LITE_ERR_ALLOC


@pytest.mark.parametrize("heads_total,code", [(2, liteattn.LITE_ERR_INVALID_ARG), (-1, liteattn.LITE_ERR_INVALID_ARG),
                                              (3, liteattn.LITE_ERR_ALLOC), (0, liteattn.LITE_ERR_ALLOC),
                                              (40, liteattn.LITE_ERR_ALLOC)])
def test_plan_heads_total_checks(lib, monkeypatch, heads_total, code):
    # a head range needs heads_total >= H (0 = H); valid ones reach the injected allocation fault
    monkeypatch.setenv("LITE_ATTN_FAULT", "alloc")
    arr = (ctypes.c_float * 1)(-1.0)
    h = ctypes.c_void_p()
    for layout in (liteattn.LITE_LAYOUT_BHND, liteattn.LITE_LAYOUT_BNHD):
        assert lib.lite_attn_plan_create_ex(ctypes.byref(h), 2, 3, 1000, 64, 64, 64, arr, 1, layout,
                                            heads_total) == code


@pytest.mark.parametrize("kw", [dict(heads_total=4, head_offset=2), dict(heads_total=2), dict(head_offset=-1)])
def test_plan_object_rejects_head_ranges_outside_the_tensors(lib, kw):
    with pytest.raises(ValueError):
        liteattn.Plan(1, 3, 64, 64, 64, 64, [-1.0], **kw)


@pytest.mark.parametrize("lens,code", [((1000, 0, 5), liteattn.LITE_ERR_INVALID_ARG),
                                       ((-3,), liteattn.LITE_ERR_INVALID_ARG),
                                       ((1 << 21, 5), liteattn.LITE_ERR_UNSUPPORTED),
                                       ((1000, 300, 1500), liteattn.LITE_ERR_ALLOC)])
def test_varlen_plan_checks(lib, monkeypatch, lens, code):
    monkeypatch.setenv("LITE_ATTN_FAULT", "alloc")       # valid ones reach the injected allocation fault
    arr = (ctypes.c_float * 1)(-1.0)
    h = ctypes.c_void_p()
    lens_c = (ctypes.c_int32 * len(lens))(*lens)
    assert lib.lite_attn_plan_create_varlen(ctypes.byref(h), len(lens), 3, lens_c, 64, 64, 64, arr, 1) == code
    assert lib.lite_attn_plan_create_varlen(ctypes.byref(h), 1, 3, None, 64, 64, 64, arr, 1) == \
        liteattn.LITE_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(seq_lens=[]), dict(seq_lens=[5, 0]), dict(seq_lens=[5, 6], N=7),
                                dict(seq_lens=[5, 6], heads_total=4)])
def test_varlen_plan_object_checks(lib, kw):
    args = dict(B=None, H=2, N=None, d=64, Br=64, Bc=64, taus=[-1.0])
    args.update(kw)
    with pytest.raises(ValueError):
        liteattn.Plan(**args)


def test_plan_object_rejects_unknown_layout_name(lib):
    with pytest.raises(ValueError):
        liteattn.Plan(1, 1, 64, 64, 64, 64, [-1.0], layout="nbhd")


def test_minus_infinity_threshold_passes_validation(lib, monkeypatch):
    # -inf is a valid threshold; the injected allocation fault proves validation passed
    monkeypatch.setenv("LITE_ATTN_FAULT", "alloc")
    rc, h = _create(taus=(-math.inf, -1.0))
    assert rc == liteattn.LITE_ERR_ALLOC


def test_host_fault_injection_alloc(lib, monkeypatch):
    monkeypatch.setenv("LITE_ATTN_FAULT", "alloc")
    rc, h = _create()
    assert rc == liteattn.LITE_ERR_ALLOC and not h.value
    with pytest.raises(liteattn.LiteAttnError) as ei:
        liteattn.Plan(1, 1, 128, 64, 64, 64, [-1.0])
    assert ei.value.code == liteattn.LITE_ERR_ALLOC


def test_null_handles_rejected(lib):
    assert lib.lite_attn_plan_destroy(None) == liteattn.LITE_OK
    assert lib.lite_attn_mask_destroy(None) == liteattn.LITE_OK
    assert lib.lite_attn_mask_reset(None, None) == liteattn.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_step(None, None, None, None, None, None, None, 0, None) == liteattn.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_stats(None, None, None) == liteattn.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_plan_info(None, None, None, None, None) == liteattn.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_mask_create(None, None) == liteattn.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_timing_enable(None, 1) == liteattn.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_launch_count() >= 0


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(liteattn, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        liteattn.load(str(tmp_path / "nope.so"))


@pytest.mark.parametrize("args,code", [
    # (bits, B, H, N, Br, Bc, list, cnt, order, live_total)
    ((None, 1, 1, 1000, 64, 64, 8, 8, 8, 8), liteattn.LITE_ERR_INVALID_ARG),
    ((8, 1, 1, 1000, 64, 64, None, 8, 8, 8), liteattn.LITE_ERR_INVALID_ARG),
    ((8, 1, 1, 1000, 64, 64, 8, None, 8, 8), liteattn.LITE_ERR_INVALID_ARG),
    ((8, 1, 1, 1000, 64, 64, 8, 8, None, 8), liteattn.LITE_ERR_INVALID_ARG),
    ((8, 1, 1, 1000, 64, 64, 8, 8, 8, None), liteattn.LITE_ERR_INVALID_ARG),
    ((8, 0, 1, 1000, 64, 64, 8, 8, 8, 8), liteattn.LITE_ERR_INVALID_ARG),
    ((8, 1, 0, 1000, 64, 64, 8, 8, 8, 8), liteattn.LITE_ERR_INVALID_ARG),
    ((8, 1, 1, 1000, 96, 96, 8, 8, 8, 8), liteattn.LITE_ERR_UNSUPPORTED),
    ((8, 1, 1, 1000, 64, 128, 8, 8, 8, 8), liteattn.LITE_ERR_UNSUPPORTED),
    ((8, 1, 1, 0, 64, 64, 8, 8, 8, 8), liteattn.LITE_ERR_UNSUPPORTED),
    ((8, 1, 1, (1 << 20) + 1, 64, 64, 8, 8, 8, 8), liteattn.LITE_ERR_UNSUPPORTED),
    # more query-tile pairs than the library's fixed scratch holds
    ((8, 64, 64, 1 << 20, 128, 128, 8, 8, 8, 8), liteattn.LITE_ERR_UNSUPPORTED),
    ((8, 1, 4 * 65536 // 2 + 1, 256, 128, 128, 8, 8, 8, 8), liteattn.LITE_ERR_UNSUPPORTED),
])
def test_noalloc_compaction_argument_checks(lib, args, code):
    """The allocation-free compaction validates its arguments on the host and
    returns before any device call; none of these pointers is dereferenced."""
    bits, B, H, N, Br, Bc, lst, cnt, order, live = args
    rc = lib.lite_attn_compact_noalloc(bits, B, H, N, Br, Bc, lst, cnt, order, live, None)
    assert rc == code


def test_noalloc_pair_limit_matches_the_header():
    text = open(os.path.join(ROOT, "include", "liteattn.h")).read()
    m = re.search(r"#define\s+LITE_NOALLOC_MAX_PAIRS\s+(\d+)", text)
    assert m and int(m.group(1)) == 65536


@pytest.mark.parametrize("ps,code", [((0.0,), liteattn.LITE_ERR_INVALID_ARG), ((-0.5,), liteattn.LITE_ERR_INVALID_ARG),
                                     ((1.5,), liteattn.LITE_ERR_INVALID_ARG),
                                     ((float("nan"),), liteattn.LITE_ERR_INVALID_ARG),
                                     ((0.9, 0.0), liteattn.LITE_ERR_INVALID_ARG),
                                     ((1.0,), liteattn.LITE_ERR_ALLOC), ((0.5, 0.99, 1.0), liteattn.LITE_ERR_ALLOC)])
def test_recall_plan_checks(lib, monkeypatch, ps, code):
    # a recall target must lie in (0, 1]; valid schedules reach the injected allocation fault
    monkeypatch.setenv("LITE_ATTN_FAULT", "alloc")
    arr = (ctypes.c_float * len(ps))(*ps)
    h = ctypes.c_void_p()
    for layout in (liteattn.LITE_LAYOUT_BHND, liteattn.LITE_LAYOUT_BNHD):
        assert lib.lite_attn_plan_create_recall(ctypes.byref(h), 1, 2, 1000, 128, 128, 128, arr, len(ps), layout,
                                                0) == code
        assert not h.value
    # thresholds are not recall targets: -1 is a valid tau but not a valid p
    bad = (ctypes.c_float * 1)(-1.0)
    assert lib.lite_attn_plan_create_recall(ctypes.byref(h), 1, 2, 1000, 128, 128, 128, bad, 1, 0, 0) == \
        liteattn.LITE_ERR_INVALID_ARG


def test_plan_object_predicate_checks(lib):
    with pytest.raises(ValueError):
        liteattn.Plan(1, 1, 64, 64, 64, 64, [0.9], predicate="top-p")
    with pytest.raises(ValueError):
        liteattn.Plan(None, 2, None, 64, 64, 64, [0.9], seq_lens=[100, 200], predicate="recall")
    assert lib.lite_attn_plan_predicate(None, ctypes.byref(ctypes.c_int())) == liteattn.LITE_ERR_INVALID_ARG


@pytest.mark.parametrize("opts,dims,code", [
    (dict(pair_stride=-1), (128, 128, 128), liteattn.LITE_ERR_INVALID_ARG),
    (dict(pair_stride=2), (64, 64, 64), liteattn.LITE_ERR_UNSUPPORTED),
    (dict(pair_stride=12), (128, 128, 128), liteattn.LITE_ERR_ALLOC),
    (dict(pair_stride=0), (64, 64, 64), liteattn.LITE_ERR_ALLOC),
    (dict(predicate=2), (128, 128, 128), liteattn.LITE_ERR_INVALID_ARG),
    (dict(predicate=liteattn.LITE_PRED_RECALL, pair_stride=3, layout=liteattn.LITE_LAYOUT_BNHD), (128, 128, 128),
     liteattn.LITE_ERR_ALLOC),
])
def test_plan_options_checks(lib, monkeypatch, opts, dims, code):
    # valid option sets reach the injected allocation fault
    monkeypatch.setenv("LITE_ATTN_FAULT", "alloc")
    o = liteattn.PlanOptions(opts.get("layout", 0), opts.get("heads_total", 0), opts.get("predicate", 0),
                             opts.get("pair_stride", 0))
    arr = (ctypes.c_float * 1)(0.9 if opts.get("predicate") == liteattn.LITE_PRED_RECALL else -1.0)
    h = ctypes.c_void_p()
    d, br, bc = dims
    assert lib.lite_attn_plan_create_opts(ctypes.byref(h), 1, 2, 1000, d, br, bc, arr, 1, ctypes.byref(o)) == code
    assert lib.lite_attn_plan_create_opts(ctypes.byref(h), 1, 2, 1000, d, br, bc, arr, 1, None) == \
        liteattn.LITE_ERR_INVALID_ARG


def test_plan_object_pair_stride_checks(lib):
    with pytest.raises(ValueError):
        liteattn.Plan(None, 2, None, 128, 128, 128, [-1.0], seq_lens=[100, 200], pair_stride=4)
