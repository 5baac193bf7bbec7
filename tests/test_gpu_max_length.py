"""GPU: the longest sequences a plan accepts.

A plan takes N up to 2^20 tokens.  With 64-wide tiles that is 16384 key tiles
per mask row, which fills the attention kernel's shared-memory bitmap (512
words per query tile) and gives compaction its longest lists.  The d = 128
case is just below the limit, with a ragged last tile (80 valid rows and
columns).  Each case runs two steps on locality-structured inputs: step 0 from
an all-live mask, step 1 from the mask step 0 propagated.  Sampled work items
(always including the head's first and last query tiles) are compared element
by element with the oracle, and the step's counters with the mask bits.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from temporal_block_sparse_sm_b200 import liteattn, synthetic
from tests.parity import check_step, pick_items

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


@pytest.mark.parametrize("d,grid", [(64, (16, 256, 256)), (128, (15, 260, 268))],
                         ids=["d64-N1048576", "d128-N1045200"])
def test_longest_sequences_match_the_oracle(d, grid):
    N = grid[0] * grid[1] * grid[2]
    assert N <= 1 << 20
    T = 2
    cfg = synthetic.WorkloadConfig(f"max-N{N}-d{d}", 1, 1, N, d, d, d, grid, T, 0.02, 0.0,
                                   schedule=("const", math.log(1e-3), math.log(1e-3)))
    plan = liteattn.Plan(cfg.B, cfg.H, N, d, d, d, cfg.taus())
    assert plan.Tk == -(-N // d)
    if d == 64:
        assert plan.W == 512, "N = 2^20 with 64-wide tiles fills the kernel's bitmap"
    else:
        assert N % d == 80
    mask = plan.mask()
    wl = synthetic.Workload(cfg, seed=3, device="cuda")
    o = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        q, k, v = wl.inputs(t)
        bits_in = mask.export_bits()
        plan.step(q, k, v, o, mask, mask, t)
        bits_out = mask.export_bits()
        st = plan.stats(mask)
        assert st["device_status"] == 0
        assert st["live_in"] == int(oracle.bits_to_bool(bits_in, plan.Tk).sum())
        assert st["live_out"] == int(oracle.bits_to_bool(bits_out, plan.Tk).sum())
        items = pick_items(cfg.B, cfg.H, plan.Tq, 12, 4000 + t)
        r = check_step(q, k, v, o, bits_in, bits_out, B=cfg.B, H=cfg.H, N=N, d=d, Br=d, Bc=d,
                       tau=plan.taus[t], items=items, step=t)
        print(cfg.name, "step", t, "skip", round(st["skip_fraction"], 4), r)
        if t == 0:
            assert st["skip_fraction"] > 0.05, "the locality inputs should kill tiles at this length"
