"""GPU tests of the C ABI's argument checks, fault paths and timing hooks."""
from __future__ import annotations

import ctypes
import math

import numpy as np
import pytest
import torch

from temporal_block_sparse_sm_b200 import liteattn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from temporal_block_sparse_sm_b200 import build
    build.build()
    liteattn.load()


def _setup(N=512, d=64, T=2):
    plan = liteattn.Plan(1, 2, N, d, d, d, [-1.0] * T)
    m = plan.mask()
    q = torch.randn(1, 2, N, d, device="cuda").to(torch.bfloat16)
    return plan, m, q, q.clone(), q.clone(), torch.empty_like(q)


def _raw_step(plan, q, k, v, o, mi, mo, step):
    return liteattn.load().lite_attn_step(plan.handle, q, k, v, o, mi.handle, mo.handle, step,
                                          torch.cuda.current_stream().cuda_stream)


def test_step_rejects_bad_pointers():
    plan, m, q, k, v, o = _setup()
    p = lambda t: t.data_ptr()
    ok = _raw_step(plan, p(q), p(k), p(v), p(o), m, m, 0)
    assert ok == liteattn.LITE_OK
    INV = liteattn.LITE_ERR_INVALID_ARG
    assert _raw_step(plan, None, p(k), p(v), p(o), m, m, 0) == INV
    assert _raw_step(plan, p(q) + 2, p(k), p(v), p(o), m, m, 0) == INV          # misaligned
    # an exact 64 KiB allocation is smaller than the 128 KiB the step reads
    from cuda.bindings import runtime as cudart
    err, small = cudart.cudaMalloc(64 * 1024)
    assert err == cudart.cudaError_t.cudaSuccess
    try:
        assert _raw_step(plan, int(small), p(k), p(v), p(o), m, m, 0) == INV    # allocation too small
    finally:
        cudart.cudaFree(small)
    host = torch.empty_like(q, device="cpu")
    assert _raw_step(plan, host.data_ptr(), p(k), p(v), p(o), m, m, 0) == INV  # host memory
    assert _raw_step(plan, p(q), p(k), p(v), p(q), m, m, 0) == INV              # o aliases q
    assert _raw_step(plan, p(q), p(k), p(v), p(o), m, m, 2) == INV              # step >= T
    assert _raw_step(plan, p(q), p(k), p(v), p(o), m, m, -1) == INV
    other = liteattn.Plan(1, 2, 512, 64, 64, 64, [-1.0])
    om = other.mask()
    assert _raw_step(plan, p(q), p(k), p(v), p(o), om, m, 0) == liteattn.LITE_ERR_PLAN_MISMATCH
    assert _raw_step(plan, p(q), p(k), p(v), p(o), m, om, 0) == liteattn.LITE_ERR_PLAN_MISMATCH
    with pytest.raises(liteattn.LiteAttnError):
        plan.stats(om)
    torch.cuda.synchronize()


def test_python_layer_checks_tensors():
    plan, m, q, k, v, o = _setup()
    with pytest.raises(ValueError):
        plan.step(q.float(), k, v, o, m, m, 0)
    with pytest.raises(ValueError):
        plan.step(q[:, :1], k, v, o, m, m, 0)
    with pytest.raises(ValueError):
        plan.step(q.transpose(2, 3), k, v, o, m, m, 0)


def test_fault_injection_paths(monkeypatch):
    plan, m, q, k, v, o = _setup()
    monkeypatch.setenv("LITE_ATTN_FAULT", "launch")
    before = liteattn.lite_attn_launch_count()
    with pytest.raises(liteattn.LiteAttnError) as ei:
        plan.step(q, k, v, o, m, m, 0)
    assert ei.value.code == liteattn.LITE_ERR_CUDA
    assert liteattn.lite_attn_launch_count() == before, "nothing may launch under an injected launch fault"
    monkeypatch.setenv("LITE_ATTN_FAULT", "status")
    st = plan.stats(m, check=False)
    assert st["rc"] == liteattn.LITE_ERR_DEVICE_TIMEOUT and st["device_status"] == liteattn.LITE_ERR_DEVICE_TIMEOUT
    monkeypatch.delenv("LITE_ATTN_FAULT")
    st = plan.stats(m)
    assert st["device_status"] == 0


def test_timing_and_launch_counter():
    plan, m, q, k, v, o = _setup(N=4096, d=128)
    plan.timing(True)
    n0 = liteattn.lite_attn_launch_count()
    for t in range(2):
        plan.step(q, k, v, o, m, m, t)
    attn_ms, step_ms, n = plan.timing_read()
    assert n == 2 and 0 < attn_ms <= step_ms
    assert liteattn.lite_attn_launch_count() - n0 == 4   # attention + compaction per step
    plan.timing(False)


def test_two_plans_on_two_streams_match_their_sequential_runs():
    """Plans share no device state: two plans stepping at the same time on two
    streams give, bit for bit, the outputs and masks of running them one after
    the other (the kernels are deterministic)."""
    shapes = [(1, 4, 4096, 128), (2, 3, 3000, 64)]
    T = 3
    g = torch.Generator(device="cuda").manual_seed(8)
    inputs = [[tuple((1.5 * torch.randn(B, H, N, d, generator=g, device="cuda")).to(torch.bfloat16)
                     for _ in range(3)) for _ in range(T)] for (B, H, N, d) in shapes]
    taus = [math.log(1e-3)] * T

    def run(streams):
        plans = [liteattn.Plan(B, H, N, d, d, d, taus) for (B, H, N, d) in shapes]
        masks = [p.mask() for p in plans]
        outs = [[torch.empty(p.shape, dtype=torch.bfloat16, device="cuda") for _ in range(T)] for p in plans]
        torch.cuda.synchronize()
        for t in range(T):
            for i, p in enumerate(plans):
                s = streams[i] if streams else None
                q, k, v = inputs[i][t]
                p.step(q, k, v, outs[i][t], masks[i], masks[i], t, s)
        torch.cuda.synchronize()
        return outs, [m.export_bits() for m in masks], [p.stats(m)["live_out"] for p, m in zip(plans, masks)]

    seq_o, seq_b, seq_live = run(None)
    con_o, con_b, con_live = run([torch.cuda.Stream(), torch.cuda.Stream()])
    for i in range(len(shapes)):
        for t in range(T):
            assert torch.equal(con_o[i][t].view(torch.int16), seq_o[i][t].view(torch.int16)), (i, t)
        assert np.array_equal(con_b[i], seq_b[i])
        assert con_live[i] == seq_live[i]


def test_a_plan_runs_on_its_own_device_whatever_the_current_device():
    """A plan belongs to the device current at its creation.  Driven while another
    device is current (the last visible device against device 0, where two are
    visible; the same device otherwise), every call runs on the plan's device,
    leaves the caller's current device unchanged, and gives bit for bit the
    results of driving the plan with its own device current."""
    last = torch.cuda.device_count() - 1
    B, H, N, d = 1, 2, 1000, 64
    taus = [math.log(1e-2)] * 2
    with torch.cuda.device(last):
        g = torch.Generator(device=f"cuda:{last}").manual_seed(12)
        q, k, v = ((1.5 * torch.randn(B, H, N, d, generator=g, device=f"cuda:{last}")).to(torch.bfloat16)
                   for _ in range(3))
        ref_plan = liteattn.Plan(B, H, N, d, d, d, taus)
        ref_mask = ref_plan.mask()
        ref_o = torch.empty_like(q)
        for t in range(2):
            ref_plan.step(q, k, v, ref_o, ref_mask, ref_mask, t)
        ref_bits = ref_mask.export_bits()
        plan = liteattn.Plan(B, H, N, d, d, d, taus)
        mask = plan.mask()
        o = torch.empty_like(q)
    assert plan.device == last
    torch.cuda.set_device(0)
    for t in range(2):
        plan.step(q, k, v, o, mask, mask, t)
        assert torch.cuda.current_device() == 0
    st = plan.stats(mask)
    bits = mask.export_bits()
    assert torch.cuda.current_device() == 0
    torch.cuda.synchronize(last)
    assert st["device_status"] == 0
    assert np.array_equal(bits, ref_bits)
    assert torch.equal(o.view(torch.int16), ref_o.view(torch.int16))
