"""GPU: plans over a range of heads (heads_total > H).

Work items are independent across heads, so plans over disjoint head ranges
of the same tensors must reproduce one plan over all heads bit for bit:
outputs, and the mask rows of their heads, step after step, in both tensor
layouts.  A range plan must not touch the other heads' output memory.  Each
range plan's heads are also checked against the oracle run on that head slice
alone, so an addressing error shared by range and full plans cannot pass.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import liteattn, synthetic
from tests.helpers import locality_qkv
from tests.parity import check_step, pick_items

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


def _layout(x: torch.Tensor, layout: str) -> torch.Tensor:
    return x.transpose(1, 2).contiguous() if layout == "bnhd" else x


CASES = [("c2", None, [(0, 5), (5, 12)]),
         (None, (2, 3, 1000, 64), [(0, 1), (1, 3)]),
         (None, (3, 4, 300, 128), [(0, 1), (1, 2), (2, 3), (3, 4)])]


@pytest.mark.parametrize("layout", ["bhnd", "bnhd"])
@pytest.mark.parametrize("cfg_name,shape,ranges", CASES)
def test_head_shards_reproduce_the_full_plan(layout, cfg_name, shape, ranges):
    if cfg_name:
        cfg = synthetic.CONFIGS[cfg_name]
        B, H, N, d = cfg.B, cfg.H, cfg.N, cfg.d
        T = 3
        taus = cfg.taus()[:T]
        wl = synthetic.Workload(cfg, seed=0, device="cuda")
        inputs = [tuple(_layout(x, layout) for x in wl.inputs(t)) for t in range(T)]
    else:
        B, H, N, d = shape
        T = 3
        taus = [math.log(1e-2)] * T
        # the workloads' seeded locality generator on a line of N tokens
        inputs = [tuple(_layout(x, layout) for x in locality_qkv(B, H, N, d, seed=11, t=t)) for t in range(T)]
    full = liteattn.Plan(B, H, N, d, d, d, taus, layout=layout)
    fmask = full.mask()
    shards = [liteattn.Plan(B, h1 - h0, N, d, d, d, taus, layout=layout, heads_total=H, head_offset=h0)
              for h0, h1 in ranges]
    smasks = [p.mask() for p in shards]
    o_full = torch.empty(full.shape, dtype=torch.bfloat16, device="cuda")
    o_shard = torch.full(full.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        q, k, v = inputs[t]
        full.step(q, k, v, o_full, fmask, fmask, t)
        ins = []
        for p, m in zip(shards, smasks):
            ins.append(m.export_bits())
            p.step(q, k, v, o_shard, m, m, t)
        torch.cuda.synchronize()
        bhnd = lambda x: x.transpose(1, 2) if layout == "bnhd" else x
        for (h0, h1), p, m, b_in in zip(ranges, shards, smasks, ins):
            sl = lambda x: bhnd(x)[:, h0:h1].contiguous()
            items = pick_items(B, h1 - h0, p.Tq, 48, 100 * t + h0)
            check_step(sl(q), sl(k), sl(v), sl(o_shard), b_in, m.export_bits(), B=B, H=h1 - h0, N=N, d=d, Br=d,
                       Bc=d, tau=p.taus[t], items=items, step=t)
        assert torch.equal(o_shard.view(torch.int16), o_full.view(torch.int16)), f"step {t}: outputs differ"
        fbits = fmask.export_bits().reshape(B, H, full.Tq, full.W)
        for (h0, h1), p, m in zip(ranges, shards, smasks):
            got = m.export_bits().reshape(B, h1 - h0, p.Tq, p.W)
            assert np.array_equal(got, fbits[:, h0:h1]), f"step {t}: mask rows of heads {h0}..{h1} differ"
    live = sum(p.stats(m)["live_out"] for p, m in zip(shards, smasks))
    assert live == full.stats(fmask)["live_out"]


@pytest.mark.parametrize("layout", ["bhnd", "bnhd"])
def test_a_head_range_writes_only_its_heads(layout):
    B, H, N, d = 2, 3, 500, 64
    g = torch.Generator(device="cuda").manual_seed(3)
    q, k, v = (_layout(torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16), layout)
               for _ in range(3))
    plan = liteattn.Plan(B, 2, N, d, d, d, [-1.0], layout=layout, heads_total=H, head_offset=1)
    m = plan.mask()
    o = torch.full(plan.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    plan.step(q, k, v, o, m, m, 0)
    torch.cuda.synchronize()
    head0 = o[:, 0] if layout == "bhnd" else o[:, :, 0]
    rest = o[:, 1:] if layout == "bhnd" else o[:, :, 1:]
    assert torch.isnan(head0).all(), "a head outside the plan's range was written"
    assert torch.isfinite(rest).all(), "the plan's heads were not all written"
