"""GPU: variable-length batches (lite_attn_plan_create_varlen).

Sequences attend within themselves, so a variable-length plan over packed
[total][H][d] tensors must reproduce, bit for bit, separate fixed-length plans
run on each sequence alone: outputs, and the mask rows of each sequence (its
missing query-tile rows and key-tile bits stay dead), step after step.  Each
sequence's slice is also checked against the oracle run on that sequence alone
(every work item, every step), so an addressing error shared by both plan kinds
cannot pass.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import liteattn
from tests.helpers import locality_qkv
from tests.parity import check_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


def _seq_inputs(lens, H, d, T, seed):
    """Per step: per-sequence [1, N_b, H, d] tensors (token-major) from the workloads' seeded
    locality generator on a line of N_b tokens (v at unit scale, as the workloads')."""
    out = []
    for t in range(T):
        step = []
        for b, n in enumerate(lens):
            q, k, v = locality_qkv(1, H, n, d, seed=seed + b, t=t)
            step.append(tuple(x.transpose(1, 2).contiguous() for x in (q, k, v)))
        out.append(step)
    return out


@pytest.mark.parametrize("lens,H,d", [((1000, 300, 1500, 64), 3, 64), ((700, 1300, 129), 2, 128), ((1,), 2, 64),
                                        ((1, 2000, 1, 65), 2, 128), ((1, 1, 129), 3, 64)])
def test_varlen_matches_per_sequence_plans(lens, H, d):
    T = 3
    taus = [math.log(1e-2)] * T
    inputs = _seq_inputs(lens, H, d, T, seed=sum(lens))
    vp = liteattn.Plan(None, H, None, d, d, d, taus, seq_lens=lens)
    vm = vp.mask()
    assert vp.shape == (sum(lens), H, d)
    seq = [liteattn.Plan(1, H, n, d, d, d, taus, layout="bnhd") for n in lens]
    sm = [p.mask() for p in seq]
    off = np.concatenate([[0], np.cumsum(lens)])
    st0 = vp.stats(vm)
    assert st0["tiles_total"] == sum(p.stats(m)["tiles_total"] for p, m in zip(seq, sm))
    assert st0["live_out"] == st0["tiles_total"]           # reset: only existing tiles live
    for t in range(T):
        q, k, v = (torch.cat([x[i][0] for x in inputs[t]], dim=0) for i in range(3))
        o = torch.full((sum(lens), H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        bits_in = vm.export_bits().reshape(len(lens), H, vp.Tq, vp.W)
        vp.step(q, k, v, o, vm, vm, t)
        bits = vm.export_bits().reshape(len(lens), H, vp.Tq, vp.W)
        for b, n in enumerate(lens):
            # the oracle on sequence b alone: its [1, H, n, d] slice and its own mask rows
            Tq_b, Tk_b = -(-n // d), -(-n // d)
            W_b = -(-Tk_b // 32)
            sl = slice(int(off[b]), int(off[b + 1]))
            qs, ks, vs, os_ = (x[sl].permute(1, 0, 2).unsqueeze(0).contiguous() for x in (q, k, v, o))
            rin = np.ascontiguousarray(bits_in[b, :, :Tq_b, :W_b]).reshape(H * Tq_b, W_b)
            rout = np.ascontiguousarray(bits[b, :, :Tq_b, :W_b]).reshape(H * Tq_b, W_b)
            check_step(qs, ks, vs, os_, rin, rout, B=1, H=H, N=n, d=d, Br=d, Bc=d, tau=vp.taus[t],
                       items=np.arange(H * Tq_b), step=t)
        for b, (p, m) in enumerate(zip(seq, sm)):
            ob = torch.empty(1, lens[b], H, d, dtype=torch.bfloat16, device="cuda")
            p.step(*inputs[t][b], ob, m, m, t)
            torch.cuda.synchronize()
            assert torch.equal(o[off[b]:off[b + 1]].view(torch.int16), ob[0].view(torch.int16)), (t, b)
            want = m.export_bits().reshape(H, p.Tq, p.W)
            assert np.array_equal(bits[b, :, : p.Tq, : p.W], want), (t, b)
            assert not bits[b, :, p.Tq:].any() and not bits[b, :, :, p.W:].any()
        live = sum(p.stats(m)["live_out"] for p, m in zip(seq, sm))
        assert vp.stats(vm)["live_out"] == live


def test_equal_lengths_match_a_batched_plan():
    B, H, N, d = 3, 2, 500, 64
    g = torch.Generator(device="cuda").manual_seed(2)
    q, k, v = ((2.0 * torch.randn(B, N, H, d, generator=g, device="cuda")).to(torch.bfloat16) for _ in range(3))
    taus = [math.log(1e-2)]
    bp = liteattn.Plan(B, H, N, d, d, d, taus, layout="bnhd")
    vp = liteattn.Plan(None, H, None, d, d, d, taus, seq_lens=[N] * B)
    bm, vm = bp.mask(), vp.mask()
    ob = torch.empty_like(q)
    ov = torch.empty(B * N, H, d, dtype=torch.bfloat16, device="cuda")
    bp.step(q, k, v, ob, bm, bm, 0)
    vp.step(q.reshape(B * N, H, d), k.reshape(B * N, H, d), v.reshape(B * N, H, d), ov, vm, vm, 0)
    torch.cuda.synchronize()
    assert torch.equal(ov.view(torch.int16), ob.reshape(B * N, H, d).view(torch.int16))
    assert np.array_equal(vm.export_bits(), bm.export_bits())


def test_varlen_import_rejects_tiles_a_sequence_lacks():
    vp = liteattn.Plan(None, 2, None, 64, 64, 64, [-1.0], seq_lens=[1000, 100])
    m = vp.mask()
    bits = m.export_bits()                                   # all existing tiles live
    m.import_bits(bits)                                      # accepted
    bad = bits.reshape(2, 2, vp.Tq, vp.W).copy()
    bad[1, 0, vp.Tq - 1, 0] = 1                              # a query tile sequence 1 does not have
    with pytest.raises(liteattn.LiteAttnError):
        m.import_bits(bad.reshape(vp.R, vp.W))
    bad = bits.reshape(2, 2, vp.Tq, vp.W).copy()
    bad[1, 0, 0, 0] |= np.uint32(1 << 5)                     # key tile 5 of a 2-tile sequence
    with pytest.raises(liteattn.LiteAttnError):
        m.import_bits(bad.reshape(vp.R, vp.W))
