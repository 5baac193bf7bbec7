"""GPU: the kernel's timeout path.

Every wait in the attention kernel is bounded.  With LITE_ATTN_FAULT=device_wait
the first CTA's first softmax warp waits on a barrier that nothing arrives on,
so its wait runs out (after about 2 s), the CTA takes its abort path (keeps its
named barriers balanced, drains its copies and MMAs, frees Tensor Memory) and
the plan's status word reads LITE_ERR_DEVICE_TIMEOUT.  The context stays
usable: a new plan then runs a correct step.  No fault, trap or endless loop
is involved.
"""
from __future__ import annotations

import math
import time

import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import liteattn, synthetic
from tests.parity import check_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


@pytest.mark.parametrize("d", [64, 128])
def test_wait_that_runs_out_reports_timeout_and_leaves_the_context_usable(monkeypatch, d):
    B, H, N = 1, 2, 1024
    g = torch.Generator(device="cuda").manual_seed(17)
    q, k, v = (torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
    taus = [math.log(1e-4)]

    plan = liteattn.Plan(B, H, N, d, d, d, taus)
    mask = plan.mask()
    o = torch.empty_like(q)
    torch.cuda.synchronize()
    monkeypatch.setenv("LITE_ATTN_FAULT", "device_wait")
    t0 = time.time()
    plan.step(q, k, v, o, mask, mask, 0)        # enqueues; the failure is reported by the device
    monkeypatch.delenv("LITE_ATTN_FAULT")
    torch.cuda.synchronize()
    waited = time.time() - t0
    st = plan.stats(mask, check=False)
    assert st["rc"] == liteattn.LITE_ERR_DEVICE_TIMEOUT
    assert st["device_status"] == liteattn.LITE_ERR_DEVICE_TIMEOUT
    assert 1.0 < waited < 60.0, waited
    # the status is sticky for that plan
    plan.step(q, k, v, o, mask, mask, 0)
    assert plan.stats(mask, check=False)["device_status"] == liteattn.LITE_ERR_DEVICE_TIMEOUT

    # the context still works: a new plan computes a correct step
    plan2 = liteattn.Plan(B, H, N, d, d, d, taus)
    mask2 = plan2.mask()
    bits_in = mask2.export_bits()
    o2 = torch.full_like(q, float("nan"))
    plan2.step(q, k, v, o2, mask2, mask2, 0)
    st2 = plan2.stats(mask2)
    assert st2["device_status"] == 0
    check_step(q, k, v, o2, bits_in, mask2.export_bits(), B=B, H=H, N=N, d=d, Br=d, Bc=d, tau=taus[0],
               items=np.arange(plan2.R), step=0)
