"""Denoising steps whose inputs and outputs live in host memory.

A caller that keeps q, k, v in (pinned) host memory and wants each step's
output back on the host pays two PCIe transfers per step.  This helper
overlaps them with the attention: step i's inputs are copied in while step
i-1 computes, and step i-1's output is copied out while step i computes.
Three CUDA streams (copy-in, compute, copy-out) and two device buffer sets;
only the compute stream touches the plan and its mask, as the C ABI requires.
Every byte is still copied every step.  PyTorch supplies the device memory,
streams and events; the step itself is ``lite_attn_step``.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence


class HostPipeline:
    """Run ``plan.step`` over a sequence of host-resident inputs.

    ``plan``: a :class:`liteattn.Plan`; ``mask``: its mask (read and written in
    place by every step).  Host tensors should be pinned for asynchronous copies.
    """

    def __init__(self, plan, mask, device=None):
        import torch

        self.torch = torch
        self.plan, self.mask = plan, mask
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        shape = plan.shape
        mk = lambda: torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        self.dev_in = [tuple(mk() for _ in range(3)) for _ in range(2)]
        self.dev_out = [mk() for _ in range(2)]
        self.s_in = torch.cuda.Stream(self.device)
        self.s_out = torch.cuda.Stream(self.device)
        self.s_cmp = torch.cuda.current_stream(self.device)
        ev = lambda: torch.cuda.Event()
        self.in_ready, self.cmp_done, self.out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        self.started = [False, False]

    def run(self, host_inputs: Sequence[tuple], host_outputs: Sequence, steps: Sequence[int],
            before_step: Optional[Callable[[int, int], None]] = None):
        """Step i uses host_inputs[i] (q, k, v), threshold index steps[i], and writes host_outputs[i].

        before_step(i, step) runs on the compute stream before step i (e.g. a mask reset).
        Returns after enqueueing; call :meth:`finish` (or synchronise) before reading outputs."""
        torch = self.torch
        n = len(steps)
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(self.s_in):
                if self.started[b]:
                    self.s_in.wait_event(self.cmp_done[b])      # step i-2 finished reading buffer b
                for j in range(3):
                    self.dev_in[b][j].copy_(host_inputs[i][j], non_blocking=True)
                self.in_ready[b].record(self.s_in)
            self.s_cmp.wait_event(self.in_ready[b])
            if self.started[b]:
                self.s_cmp.wait_event(self.out_free[b])         # step i-2's output left buffer b
            if before_step is not None:
                before_step(i, steps[i])
            q, k, v = self.dev_in[b]
            self.plan.step(q, k, v, self.dev_out[b], self.mask, self.mask, steps[i], self.s_cmp)
            self.cmp_done[b].record(self.s_cmp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.cmp_done[b])
                host_outputs[i].copy_(self.dev_out[b], non_blocking=True)
                self.out_free[b].record(self.s_out)
            self.started[b] = True

    def finish(self):
        """Make the compute stream wait for the last output copy."""
        for b in range(2):
            if self.started[b]:
                self.s_cmp.wait_event(self.out_free[b])
