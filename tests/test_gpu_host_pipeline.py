"""GPU: host-resident steps through HostPipeline (copies overlapped with the
attention) give the same outputs and masks, bit for bit, as device-resident
steps, including across two run() calls and a mask reset mid-sequence."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import liteattn, synthetic
from temporal_block_sparse_sm_b200.host_pipeline import HostPipeline

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


@pytest.mark.parametrize("cfg_name", ["c1", "c2"])
def test_host_pipeline_matches_device_steps(cfg_name):
    cfg = synthetic.CONFIGS[cfg_name]
    T = cfg.T
    steps = [t % T for t in range(T + 3)]               # wraps into a second trajectory
    wl = synthetic.Workload(cfg, seed=3, device="cuda")
    inputs = [wl.inputs(t) for t in range(T)]

    ref_plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, cfg.taus())
    ref_mask = ref_plan.mask()
    o = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
    ref = []
    for t in steps:
        if t == 0:
            ref_mask.reset()
        q, k, v = inputs[t]
        ref_plan.step(q, k, v, o, ref_mask, ref_mask, t)
        ref.append(o.cpu())
    ref_bits = ref_mask.export_bits()

    plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, cfg.taus())
    mask = plan.mask()
    host_in = [tuple(x.cpu().pin_memory() for x in inputs[t]) for t in steps]
    host_out = [torch.full(wl.shape, float("nan"), dtype=torch.bfloat16).pin_memory() for _ in steps]
    pipe = HostPipeline(plan, mask)
    reset = lambda i, t: mask.reset() if t == 0 else None
    half = len(steps) // 2
    pipe.run(host_in[:half], host_out[:half], steps[:half], reset)
    pipe.run(host_in[half:], host_out[half:], steps[half:], reset)
    pipe.finish()
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(host_out, ref)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"step {i} differs"
    assert np.array_equal(mask.export_bits(), ref_bits)
