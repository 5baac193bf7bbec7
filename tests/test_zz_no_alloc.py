"""The allocation-free compaction entry point, checked against the mask store.

Some callers cannot call cudaMalloc: their device memory belongs to another
allocator (a framework's caching allocator or a preallocated arena), or their
serving loop must not allocate after start-up.  lite_attn_compact_noalloc
serves them: it rebuilds the compacted live lists of a caller-owned bitmask
into caller-owned buffers, with its scratch in a fixed array inside the
library.  This test feeds it the same bitmasks as a plan's mask store
(lite_attn_mask_import, which uses allocated scratch) and compares the two,
on two calls in a row with different masks, so a stale scratch array would
show.  It passes run alone or after the rest of the suite.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import liteattn, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


def _u32_tensor(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32).view(np.int32)).cuda()


@pytest.mark.parametrize("shape", [(1, 12, 8192, 128), (2, 3, 1000, 64), (1, 2, 70000, 64)])
def test_noalloc_compaction_matches_mask_store(shape):
    B, H, N, bc = shape
    plan = liteattn.Plan(B, H, N, bc, bc, bc, [-1.0])
    mask = plan.mask()
    G, Tk, R, W = plan.G, plan.Tk, plan.R, plan.W
    lst = torch.empty(G * Tk, dtype=torch.int32, device="cuda")
    cnt = torch.empty(G, dtype=torch.int32, device="cuda")
    order = torch.empty(G, dtype=torch.int32, device="cuda")
    live = torch.empty(1, dtype=torch.int64, device="cuda")
    for call, frac in enumerate((0.4, 0.9)):          # two calls in a row, different masks
        bits = synthetic.random_live_bits(R, Tk, frac, seed=31 + call, keep_first=False).numpy().astype(np.uint32)
        mask.import_bits(bits)
        ref_list, ref_cnt, ref_order = mask.export_lists()
        ref_live = plan.stats(mask)["live_out"]

        d_bits = _u32_tensor(bits)
        lst.fill_(-1)
        cnt.fill_(-1)
        order.fill_(-1)
        liteattn.lite_attn_compact_noalloc(d_bits.data_ptr(), B, H, N, bc, bc, lst.data_ptr(), cnt.data_ptr(),
                                           order.data_ptr(), live.data_ptr())
        torch.cuda.synchronize()
        got_cnt = cnt.cpu().numpy()
        got_list = lst.cpu().numpy().view(np.uint32).reshape(G, Tk)
        got_order = order.cpu().numpy()
        assert np.array_equal(got_cnt, ref_cnt), f"call {call}: counts differ"
        for g in range(G):
            assert np.array_equal(got_list[g, : got_cnt[g]], ref_list[g, : ref_cnt[g]]), (call, g)
        assert int(live.item()) == ref_live
        # the order is longest-first; pairs with equal (bucketed) counts may come in any order
        assert np.array_equal(np.sort(got_order), np.arange(G))
        keys = (got_cnt[got_order].astype(np.int64) * min(Tk + 1, 1024)) // (Tk + 1)
        assert np.all(np.diff(keys) <= 0)
        assert np.array_equal(np.sort(got_cnt[got_order]), np.sort(ref_cnt[ref_order]))


def test_noalloc_rejects_oversize_and_bad_arguments():
    lib = liteattn.load()
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    # more query-tile pairs than the fixed scratch holds
    assert lib.lite_attn_compact_noalloc(p, 64, 64, 1 << 20, 128, 128, p, p, p, p, s) == liteattn.LITE_ERR_UNSUPPORTED
    assert lib.lite_attn_compact_noalloc(p, 1, 1, 1000, 96, 96, p, p, p, p, s) == liteattn.LITE_ERR_UNSUPPORTED
    assert lib.lite_attn_compact_noalloc(None, 1, 1, 1000, 64, 64, p, p, p, p, s) == liteattn.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_compact_noalloc(p, 0, 1, 1000, 64, 64, p, p, p, p, s) == liteattn.LITE_ERR_INVALID_ARG


def test_noalloc_rejects_buffers_it_cannot_use_without_launching():
    """Too-small, overlapping or host buffers, and a stream of no device, are
    refused on the host: INVALID_ARG and no kernel launch."""
    lib = liteattn.load()
    B, H, N, bc = 2, 3, 1000, 64
    plan = liteattn.Plan(B, H, N, bc, bc, bc, [-1.0])
    G, Tk, R, W = plan.G, plan.Tk, plan.R, plan.W
    bits = torch.zeros(R * W, dtype=torch.int32, device="cuda")
    lst = torch.empty(G * Tk, dtype=torch.int32, device="cuda")
    cnt = torch.empty(G, dtype=torch.int32, device="cuda")
    order = torch.empty(G, dtype=torch.int32, device="cuda")
    live = torch.empty(1, dtype=torch.int64, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    ok = (bits.data_ptr(), B, H, N, bc, bc, lst.data_ptr(), cnt.data_ptr(), order.data_ptr(), live.data_ptr(), s)
    assert lib.lite_attn_compact_noalloc(*ok) == liteattn.LITE_OK
    torch.cuda.synchronize()
    # Buffers that are too small: exact-size allocations of their own (the check sees
    # allocation bounds, and a tensor of the caching allocator sits inside a larger one).
    from cuda.bindings import runtime as rt
    raw = []
    for nbytes in ((G * Tk - 1) * 4, (R * W - 1) * 4):
        err, ptr = rt.cudaMalloc(nbytes)
        assert err == rt.cudaError_t.cudaSuccess
        raw.append(int(ptr))
    small_list, small_bits = raw
    host = np.zeros(G * Tk, dtype=np.int32)
    bad = [
        (small_bits,) + ok[1:],                                             # bitmask one word short
        ok[:6] + (small_list,) + ok[7:],                                    # list one entry short
        ok[:6] + (host.ctypes.data,) + ok[7:],                              # host memory
        ok[:7] + (order.data_ptr(),) + ok[8:],                              # cnt aliases order
        ok[:6] + (bits.data_ptr(),) + ok[7:],                               # list overlaps the bitmask
        ok[:9] + (live.data_ptr() + 4,) + ok[10:],                          # live_total misaligned
    ]
    try:
        n0 = liteattn.lite_attn_launch_count()
        for i, args in enumerate(bad):
            assert lib.lite_attn_compact_noalloc(*args) == liteattn.LITE_ERR_INVALID_ARG, i
        assert liteattn.lite_attn_launch_count() == n0, "a refused call launched a kernel"
    finally:
        for ptr in raw:
            rt.cudaFree(ptr)


@pytest.mark.parametrize("shape", [(2, 3, 1000, 64), (1, 4, 3000, 128)])
def test_noalloc_ignores_bits_past_the_last_key_tile(shape):
    """A caller's bitmask with stray bits >= Tk in each row's last word compacts
    exactly like the same mask without them (lists never exceed Tk entries)."""
    B, H, N, bc = shape
    plan = liteattn.Plan(B, H, N, bc, bc, bc, [-1.0])
    G, Tk, R, W = plan.G, plan.Tk, plan.R, plan.W
    assert Tk % 32, "the shape must leave unused bits in the last word"
    clean = synthetic.random_live_bits(R, Tk, 0.5, seed=77, keep_first=False).numpy().astype(np.uint32)
    junk = clean.copy()
    junk[:, W - 1] |= np.uint32(~((1 << (Tk % 32)) - 1) & 0xFFFFFFFF)
    outs = []
    for bits in (clean, junk):
        lst = torch.full((G * Tk,), -1, dtype=torch.int32, device="cuda")
        cnt = torch.full((G,), -1, dtype=torch.int32, device="cuda")
        order = torch.full((G,), -1, dtype=torch.int32, device="cuda")
        live = torch.zeros(1, dtype=torch.int64, device="cuda")
        liteattn.lite_attn_compact_noalloc(_u32_tensor(bits).data_ptr(), B, H, N, bc, bc, lst.data_ptr(),
                                           cnt.data_ptr(), order.data_ptr(), live.data_ptr())
        torch.cuda.synchronize()
        outs.append((lst.cpu().numpy(), cnt.cpu().numpy(), order.cpu().numpy(), int(live.item())))
    (l0, c0, o0, v0), (l1, c1, o1, v1) = outs
    assert np.array_equal(c0, c1) and v0 == v1 and (c1 <= Tk).all()
    assert np.array_equal(np.sort(o1), np.arange(G))
    for g in range(G):
        assert np.array_equal(l0.reshape(G, Tk)[g, : c0[g]], l1.reshape(G, Tk)[g, : c1[g]])
