#!/usr/bin/env python
"""Benchmark of the LiteAttention step on B200.

One bench step = one denoising step of the workload: the attention kernel over
the live tiles of the persistent mask plus the mask compaction, through the
C ABI.  The default workload is the largest single-GPU configuration, the
720p video-DiT attention shape (B=1, H=24, N=108000 on a 30x45x80 token grid,
d=128, 50-step threshold schedule ln 1e-6 -> ln 1e-3).  The timed steps run the
schedule from its first step (mask reset to all-live, inside the timed region)
and cycle through it; the JSON line names the schedule steps they cover.  Each
schedule step has its own input tensors, created before timing.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c4] [--impl reference]
Under torchrun every rank runs its own seeded copy of the workload (head- and
batch-independent work, no data-path collective: weak scaling); rank 0
prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dense-equiv attention TFLOPS & ms/denoise-step vs skip rate; % BF16 tensor peak"
UNIT = "TFLOPS (dense-equivalent)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a float over ranks (identity when world == 1)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    QUERY = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ CPU baseline (the oracle)
# Both host legs (the GPU arm's cpu_baseline and the reference arm) time the fp64
# oracle by one rule: a seeded uniform sample of the work items (b, h, query tile)
# of schedule step 0, all-live mask, threshold tau_0; the sample size is a
# multiple of the oracle's thread count.  value = dense-equivalent FLOPs of the
# sampled items / wall time; ms_per_step is extrapolated to all B*H*Tq items.
def host_step0_bits(cfg, inputs0=None):
    """bf16 bit patterns (numpy uint16, [B, H, N, d]) of step 0's q, k, v: from
    device tensors when given, else generated on the host."""
    import numpy as np
    import torch
    if inputs0 is None:
        from temporal_block_sparse_sm_b200.synthetic import Workload
        inputs0 = Workload(cfg, seed=0, device="cpu").inputs(0)
    return tuple(x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16) for x in inputs0)


def oracle_sample(cfg, qkv_bits, n_items: int, seed: int = 0):
    """Time the oracle on n_items seeded work items of step 0 (all-live mask, tau_0).

    Returns (seconds, items, dense-equivalent flops of the sampled items, threads used)."""
    import numpy as np
    import oracle
    qh, kh, vh = qkv_bits
    Tq, Tk, W = oracle.tiles(cfg.N, cfg.Br, cfg.Bc)
    R = cfg.B * cfg.H * Tq
    rng = np.random.default_rng(seed)
    items = np.sort(rng.choice(R, size=min(n_items, R), replace=False)).astype(np.int64)
    mask_in = oracle.all_live_rows(len(items), cfg.N, cfg.Bc)
    t0 = time.perf_counter()
    oracle.step(qh, kh, vh, B=cfg.B, H=cfg.H, N=cfg.N, d=cfg.d, Br=cfg.Br, Bc=cfg.Bc, tau=cfg.taus()[0],
                items=items, mask_in=mask_in)
    dt = time.perf_counter() - t0
    flops = 0.0
    for it in items:
        i = int(it) % Tq
        rows = min(cfg.Br, cfg.N - i * cfg.Br)
        flops += 4.0 * rows * cfg.N * cfg.d
    return dt, len(items), flops, oracle.max_threads()


def sample_size(cfg, qkv_bits, target_s: float) -> int:
    """Items per sample so that one sample takes about target_s seconds: one
    calibration round of one item per thread, then whole rounds."""
    import oracle
    thr = oracle.max_threads()
    dt, n, _, _ = oracle_sample(cfg, qkv_bits, thr, seed=12345)
    rounds = max(1, int(round(target_s / max(dt, 1e-6))))
    Tq = -(-cfg.N // cfg.Br)
    return min(cfg.B * cfg.H * Tq, rounds * thr)


def cpu_baseline(cfg, qkv_bits, target_s: float = 12.0):
    n = sample_size(cfg, qkv_bits, target_s)
    dt, n, fl, thr = oracle_sample(cfg, qkv_bits, n, seed=1)
    Tq = -(-cfg.N // cfg.Br)
    R = cfg.B * cfg.H * Tq
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": f"{n} of the {R} query tiles of step 0 of {cfg.name} (seeded uniform draw, all-live "
                      f"mask, tau_0), fp64, {dt:.1f} s; ms_per_step extrapolated to all {R}",
            "extrapolated": n < R, "ms_per_step_extrapolated": dt / n * R * 1e3}


def run_reference(args, cfg):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    bits = host_step0_bits(cfg)
    # each step: one sample of about --ref-seconds / (warmup + steps) of oracle work,
    # so the whole run stays within a few minutes
    n_items = sample_size(cfg, bits, args.ref_seconds / max(1, args.steps + args.warmup))
    for s in range(args.warmup):
        oracle_sample(cfg, bits, n_items, seed=1000 + s)
    tot_t, tot_f, tot_n = 0.0, 0.0, 0
    for s in range(args.steps):
        dt, n, fl, thr = oracle_sample(cfg, bits, n_items, seed=s + 1)
        tot_t += dt
        tot_f += fl
        tot_n += n
    val = tot_f / tot_t / 1e12
    Tq = -(-cfg.N // cfg.Br)
    R = cfg.B * cfg.H * Tq
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_t / tot_n * R * 1e3, "ms_per_step_extrapolated": True,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "N": cfg.N, "d": cfg.d, "Br": cfg.Br,
                       "Bc": cfg.Bc, "layout": args.layout, "parallelism": "host threads"},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
                             "sample": f"each step: {n_items} of the {R} query tiles of step 0 of {cfg.name} "
                                       f"(seeded uniform draw, all-live mask, tau_0), fp64; ms_per_step "
                                       f"extrapolated to all {R}",
                             "extrapolated": n_items < R},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ GPU arm
# DRAM traffic of one attention launch on the bench workload, from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the hash of the kernel source (comments
# and whitespace removed) it was taken on.
NCU_TRAFFIC = {
    # profiles/lite_attn_fwd_kernel_c2_N8192_H12_d128.md: 86.76 MB read + 11.07 MB written
    ("c2-N8192-H12-d128", "68111d0684ba3ab9"): 97_830_144,
    # profiles/lite_attn_fwd_kernel_c4_N108000_H24_d128.md: one launch of schedule step 0 (all-live mask),
    # 4051.53 MB read + 660.65 MB written
    ("c4-N108000-H24-d128", "73b4489e85f2e7f3"): 4_712_184_320,
}


def code_hash(texts) -> str:
    """Hash of CUDA sources with comments and whitespace removed, so that an
    edit to comments alone keeps the key of counters taken on that code."""
    import hashlib
    import re
    h = hashlib.sha256()
    for t in texts:
        t = re.sub(r"/\*.*?\*/", " ", t, flags=re.S)
        t = re.sub(r"//[^\n]*", " ", t)
        h.update(" ".join(t.split()).encode())
    return h.hexdigest()[:16]


def kernel_hash() -> str:
    texts = []
    for fn in ("attn_kernel.cuh", "sm100_ptx.cuh"):
        with open(os.path.join(ROOT, "temporal_block_sparse_sm_b200", "csrc", fn)) as f:
            texts.append(f.read())
    return code_hash(texts)


def head_range(rank: int, world: int, H: int):
    """Heads [h0, h1) of `rank` when H heads are split over `world` ranks (sizes differ by at most 1)."""
    return rank * H // world, (rank + 1) * H // world


def step_ranges(steps) -> str:
    """'0..19' style summary of a sequence of schedule steps."""
    out, run = [], None
    for t in steps:
        if run and t == run[1] + 1:
            run[1] = t
        else:
            if run:
                out.append(run)
            run = [t, t]
    if run:
        out.append(run)
    return ",".join(f"{a}..{b}" if a != b else f"{a}" for a, b in out)


def pair_stride_of(arg, cfg) -> int:
    """--pair-stride: an integer, or 'frame' = whole query tiles per video frame of
    the workload's (frame, y, x) token grid (1 when a frame is under two tiles)."""
    if str(arg) == "frame":
        return max(1, (cfg.grid[1] * cfg.grid[2]) // cfg.Br) if cfg.Br == 128 else 1
    return int(arg)


def run_gpu(args, cfg):
    import torch
    from temporal_block_sparse_sm_b200 import build, liteattn, synthetic

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    if rank == 0:
        build.build()
    barrier(world, device)
    liteattn.load()

    T = cfg.T
    if args.shard == "heads":
        # one problem split by heads: rank r holds heads [h0, h1) of the seed-0 workload
        # (its own q, k, v, o and masks); work items are independent across heads, so
        # there is no exchange between ranks
        if world > cfg.H:
            raise SystemExit(f"--shard heads needs at most {cfg.H} ranks")
        h0, h1 = head_range(rank, world, cfg.H)
        seed = 0
    else:
        h0, h1 = 0, cfg.H
        seed = rank                     # independent replicas
    Hs = h1 - h0
    stride = pair_stride_of(args.pair_stride, cfg)
    plan = liteattn.Plan(cfg.B, Hs, cfg.N, cfg.d, cfg.Br, cfg.Bc, cfg.taus(), layout=args.layout, pair_stride=stride)
    mask = plan.mask()
    K, Wm = args.steps, args.warmup
    elem_bytes = cfg.B * Hs * cfg.N * cfg.d * 2
    step_bytes = 3 * elem_bytes
    # The warm-up and the timed steps both run the schedule from step 0, so they
    # touch schedule steps 0 .. max(W, K) - 1 (mod T).  Each gets its own inputs,
    # up to the device-memory budget; past it, step t reuses the inputs of
    # step t mod n_buf (said in the JSON line).
    touched = sorted({i % T for i in range(max(Wm, K))})
    n_buf = max(1, min(len(touched), int(args.input_budget_gb * 1e9 // step_bytes)))
    wl = synthetic.Workload(cfg, seed=seed, device=device)
    bufs = {}
    for t in touched[:n_buf]:
        xs = tuple(x[:, h0:h1].contiguous() for x in wl.inputs(t))
        if args.layout == "bnhd":   # the same values, token-major: [B, N, H, d]
            xs = tuple(x.transpose(1, 2).contiguous() for x in xs)
        bufs[t] = xs
    inputs0_bhnd = None
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        inputs0_bhnd = tuple(x.cpu() for x in wl.inputs(0))   # step 0 on the host, [B, H, N, d], for the oracle
    del wl
    torch.cuda.empty_cache()
    exact = n_buf == len(touched)
    # Timed steps must not find their inputs in L2 (126 MB): rotate over enough
    # copies of the per-step inputs to exceed twice that.
    reps = max(1, math.ceil(2 * 126e6 / (len(bufs) * step_bytes)))
    copies = [bufs] + [{t: tuple(x.clone() for x in xs) for t, xs in bufs.items()} for _ in range(reps - 1)]
    keys = sorted(bufs)
    o = torch.empty(bufs[keys[0]][0].shape, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def inputs_of(t, i):
        src = copies[(i // T) % reps]
        return src[t] if t in src else src[keys[t % len(keys)]]

    def one_step(i):
        t = i % T
        if t == 0:
            mask.reset(stream)
        q, k, v = inputs_of(t, i)
        plan.step(q, k, v, o, mask, mask, t, stream)

    for i in range(Wm):
        one_step(i)
    torch.cuda.synchronize(device)
    # the timed region starts a trajectory: mask reset, then schedule steps 0, 1, ...
    st0 = plan.stats(mask)
    plan.timing(True)
    n_launch0 = liteattn.lite_attn_launch_count()
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local)
    barrier(world, device)
    torch.cuda.synchronize(device)
    clocks.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(K):
        one_step(i)
    ev1.record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    barrier(world, device)
    launches = liteattn.lite_attn_launch_count() - n_launch0
    elapsed_ms = ev0.elapsed_time(ev1)
    attn_ms, step_ms, n_rec = plan.timing_read()
    plan.timing(False)
    st1 = plan.stats(mask)
    qk = st1["cum_qk_tiles"] - st0["cum_qk_tiles"]
    pv = st1["cum_pv_tiles"] - st0["cum_pv_tiles"]
    tile_flops = 2.0 * cfg.Br * cfg.Bc * cfg.d
    exec_flops = tile_flops * (qk + pv)
    dense_flops = 4.0 * cfg.B * Hs * cfg.N * cfg.N * cfg.d * K
    tiles_total = st1["tiles_total"]
    max_ms = max_over_ranks(elapsed_ms, world, device)
    tot_dense = sum_over_ranks(dense_flops, world, device)
    tot_exec = sum_over_ranks(exec_flops, world, device)

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timed region
    # Every step copies its q, k, v in from pinned host memory and its output back
    # out; HostPipeline overlaps those copies with the neighbouring steps' attention.
    e2e = None
    if not args.no_e2e:
        from temporal_block_sparse_sm_b200.host_pipeline import HostPipeline
        Ke = min(K, T)
        # pinned host inputs: every e2e step's own when they fit in the host budget,
        # else a ring of 3 (step t reads the ring entry t mod 3)
        e2e_steps = list(range(Ke))
        n_host = Ke if Ke * step_bytes <= args.host_budget_gb * 1e9 else min(3, Ke)
        host_ring = [tuple(x.cpu().pin_memory() for x in inputs_of(t, 0)) for t in e2e_steps[:n_host]]
        host_in = [host_ring[i % n_host] for i in range(Ke)]
        host_out = [torch.empty(o.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        pipe = HostPipeline(plan, mask, device)
        reset_at_start = lambda i, t: mask.reset(stream) if t == 0 else None
        pipe.run(host_in[:2], host_out, [0, 1], reset_at_start)     # warm the pipeline's streams and buffers
        pipe.finish()
        torch.cuda.synchronize(device)
        barrier(world, device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pipe.s_in.wait_event(e0)
        pipe.run(host_in, [host_out[i & 1] for i in range(Ke)], e2e_steps, reset_at_start)
        pipe.finish()
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
        e2e_dense = sum_over_ranks(4.0 * cfg.B * Hs * cfg.N * cfg.N * cfg.d * Ke, world, device)
        e2e = {"value": e2e_dense / (e2e_ms / 1e3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms / Ke,
               "h2d_bytes_per_step": step_bytes, "d2h_bytes_per_step": elem_bytes, "steps": Ke,
               "schedule_steps": step_ranges(e2e_steps),
               "host_inputs": ("each step's own pinned inputs" if n_host == Ke else
                               f"a ring of {n_host} pinned step inputs (steps 0..{n_host - 1}); step t reads "
                               f"entry t mod {n_host}")}
        del host_ring, host_in, host_out, pipe

    if rank == 0:
        peaks, peak_src = load_peaks()
        bf16 = float(peaks["bf16_tflops"])
        achieved = exec_flops / (attn_ms / 1e3) / 1e12 if attn_ms > 0 else 0.0
        khash = kernel_hash()
        traffic = NCU_TRAFFIC.get((cfg.name, khash)) if args.layout == "bhnd" else None
        timed_steps = [i % T for i in range(K)]
        line = {
            "metric": METRIC,
            "value": tot_dense / (max_ms / 1e3) / 1e12,
            "unit": UNIT,
            "n_gpus": world,
            "steps": K,
            "warmup": Wm,
            "ms_per_step": max_ms / K,
            "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "N": cfg.N, "d": cfg.d, "Br": cfg.Br,
                       "Bc": cfg.Bc, "T": T, "layout": args.layout, "schedule": "ln(1e-6)->ln(1e-3) log-linear" if cfg.schedule[0] ==
                       "loglinear" else f"const {cfg.schedule[1]:.3f}",
                       "timed_schedule_steps": step_ranges(timed_steps),
                       "pair_stride": stride,
                       "mask": "reset to all-live at the start of the timed steps and at every trajectory start, "
                               "AND-propagated in place",
                       "inputs": (f"each schedule step's own inputs ({len(bufs)} steps x {step_bytes / 1e9:.2f} GB, "
                                  "created before timing)" if exact else
                                  f"inputs of {n_buf} schedule steps ({step_bytes / 1e9:.2f} GB each, device budget "
                                  f"{args.input_budget_gb} GB); step t >= {n_buf} reuses step t mod {n_buf}'s"),
                       "l2": f"inputs larger than L2: {reps * len(bufs)} step buffers of {step_bytes / 1e6:.0f} MB "
                             f"rotate (126 MB L2)",
                       "parallelism": (f"heads{world} (one problem, heads split over ranks, no collective)"
                                       if args.shard == "heads" else
                                       f"dp{world} (independent seeded replicas, no collective)")},
            "executed_tflops": tot_exec / (max_ms / 1e3) / 1e12,
            "skip_fraction": 1.0 - pv / (tiles_total * K),
            "qk_skip_fraction": 1.0 - qk / (tiles_total * K),
            "pct_bf16_peak_executed": 100.0 * (exec_flops / (elapsed_ms / 1e3) / 1e12) / bf16,
            "attn_kernel_ms_per_step": attn_ms / max(n_rec, 1),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
                         "frac": achieved / bf16, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16 dense (burst)",
                         "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", bf16)),
                         "kernel": "lite_attn_fwd_kernel<128,128,128>" if cfg.d == 128 else
                                   "lite_attn_fwd_kernel<64,64,64>", "kernel_hash": khash},
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
        }
        if inputs0_bhnd is not None:   # the host baseline belongs to single-GPU runs
            line["cpu_baseline"] = cpu_baseline(cfg, host_step0_bits(cfg, inputs0_bhnd))
        print(json.dumps(line), flush=True)
    barrier(world, device)
    del bufs, copies
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ propagation-policy sweep
def run_policy_sweep(args, names, bf16):
    """Each workload's trajectory under each mask-propagation policy (propagate,
    recompute, early-only, refresh on divergence): ms per step, skip rate,
    throughput, refresh decisions, and the error of the last step's output
    against the dense (tau = -inf) output on the same inputs.  One JSON line per
    (workload, policy)."""
    import torch
    from temporal_block_sparse_sm_b200 import liteattn, synthetic
    from temporal_block_sparse_sm_b200.propagation import MaskPolicy, early_only_schedule

    def run(cfg, taus, policy, **kw):
        plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, taus,
                             pair_stride=pair_stride_of(args.pair_stride, cfg))
        pol = MaskPolicy(plan, policy, **kw)
        wl = synthetic.Workload(cfg, seed=0, device="cuda")
        o = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
        pol.start()
        ms, attn, skips, execf = 0.0, 0.0, [], 0.0
        tile_flops = 2.0 * cfg.Br * cfg.Bc * cfg.d
        for t in range(len(taus)):
            q, k, v = wl.inputs(t)
            torch.cuda.synchronize()
            s0 = plan.stats(pol.mask)
            plan.timing(True)
            pol.step(q, k, v, o, t)
            a_ms, s_ms, _ = plan.timing_read()
            ms += s_ms
            attn += a_ms
            s1 = plan.stats(pol.mask)
            execf += tile_flops * ((s1["cum_qk_tiles"] - s0["cum_qk_tiles"]) + (s1["cum_pv_tiles"] - s0["cum_pv_tiles"]))
            skips.append(s1["skip_fraction"])
        plan.timing(False)
        last = o.clone()
        pol.close()
        plan.close()
        return ms / len(taus), attn, execf, skips, pol.history, last

    for name in names:
        cfg = synthetic.CONFIGS[name]
        if name == "c5":
            continue
        T = cfg.T
        *_, dense_o = run(cfg, [-math.inf] * T, "propagate")
        every = max(2, T // 5)
        cases = [("propagate", cfg.taus(), {}), ("recompute", cfg.taus(), {}),
                 ("early", early_only_schedule(cfg.taus(), 2), {}),
                 ("refresh", cfg.taus(), {"every": every, "revive": args.revive})]
        dense = 4.0 * cfg.B * cfg.H * cfg.N * cfg.N * cfg.d
        for policy, taus, kw in cases:
            ms, attn, execf, skips, hist, last = run(cfg, taus, policy, **kw)
            err = (last.float() - dense_o.float()).abs()
            probes = [(h["t"], round(h["divergence"], 5), h["adopted"]) for h in hist if h["probe"]]
            print(json.dumps({"sweep": "policy", "workload": cfg.name, "policy": policy, **kw, "steps": T,
                              "pair_stride": pair_stride_of(args.pair_stride, cfg),
                              "ms_per_step": ms, "dense_eq_tflops": dense / (ms / 1e3) / 1e12,
                              "exec_tflops": execf / (attn / 1e3) / 1e12,
                              "pct_bf16_peak_exec": 100 * execf / (attn / 1e3) / 1e12 / bf16,
                              "skip_mean": sum(skips) / T, "skip_final": skips[-1], "probes": probes,
                              "err_vs_dense_last_max": float(err.max()), "err_vs_dense_last_mean": float(err.mean())}),
                  flush=True)
    return 0


# ------------------------------------------------------------------ calibration sweep
def run_calibration_sweep(args, names, bf16):
    """Accumulated-error calibration: choose the threshold schedule on the seed-1
    trajectory of each workload for per-step budgets that grow with the step
    (total --error-budget, relative L1 against dense), then run it in propagate
    mode on the seed-0 trajectory next to the log-linear stand-in schedule.
    One JSON line per (workload, schedule): skip, ms per step, throughput, and the
    per-step relative L1 error against dense with the budget it had."""
    import torch
    from temporal_block_sparse_sm_b200 import liteattn, synthetic
    from temporal_block_sparse_sm_b200.calibration import calibrate, error_budgets, threshold_grid

    for name in names:
        cfg = synthetic.CONFIGS[name]
        if name == "c5":
            continue
        T = cfg.T
        mk = lambda taus: liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, taus,
                                        pair_stride=pair_stride_of(args.pair_stride, cfg))
        new_o = lambda: torch.empty((cfg.B, cfg.H, cfg.N, cfg.d), dtype=torch.bfloat16, device="cuda")
        budgets = error_budgets(T, args.error_budget)
        grid_plan, dense_plan = mk(threshold_grid()), mk([-math.inf])
        cal_wl = synthetic.Workload(cfg, seed=1, device="cuda")
        t0 = time.time()
        res = calibrate(grid_plan, dense_plan, cal_wl.inputs, budgets, new_o)
        cal_s = time.time() - t0
        del cal_wl
        wl = synthetic.Workload(cfg, seed=0, device="cuda")
        for label, taus in (("calibrated", res.taus), ("loglinear", cfg.taus())):
            plan = mk(taus)
            mask, dmask = plan.mask(), dense_plan.mask()
            o, od = new_o(), new_o()
            ms, attn, execf, errs, skips = 0.0, 0.0, 0.0, [], []
            tile_flops = 2.0 * cfg.Br * cfg.Bc * cfg.d
            for t in range(T):
                q, k, v = wl.inputs(t)
                dmask.reset()
                dense_plan.step(q, k, v, od, dmask, dmask, 0)
                torch.cuda.synchronize()
                s0 = plan.stats(mask)
                plan.timing(True)
                plan.step(q, k, v, o, mask, mask, t)
                a_ms, s_ms, _ = plan.timing_read()
                plan.timing(False)
                s1 = plan.stats(mask)
                ms += s_ms
                attn += a_ms
                execf += tile_flops * ((s1["cum_qk_tiles"] - s0["cum_qk_tiles"]) +
                                       (s1["cum_pv_tiles"] - s0["cum_pv_tiles"]))
                errs.append(plan.output_error(o, od)["rel_l1"])
                skips.append(s1["skip_fraction"])
            dense = 4.0 * cfg.B * cfg.H * cfg.N * cfg.N * cfg.d
            line = {"sweep": "calibration", "workload": cfg.name, "schedule": label, "steps": T,
                    "pair_stride": pair_stride_of(args.pair_stride, cfg),
                    "error_budget_total": args.error_budget, "ms_per_step": ms / T,
                    "dense_eq_tflops": dense * T / (ms / 1e3) / 1e12,
                    "pct_bf16_peak_exec": 100 * execf / (attn / 1e3) / 1e12 / bf16,
                    "skip_mean": sum(skips) / T, "skip_final": skips[-1],
                    "taus": [round(x, 3) if math.isfinite(x) else "-inf" for x in taus],
                    "rel_l1_per_step": [float(f"{e:.3e}") for e in errs],
                    "budget_per_step": [float(f"{b:.3e}") for b in budgets],
                    "steps_over_budget": [t for t in range(T) if errs[t] > budgets[t]]}
            if label == "calibrated":
                line.update({"calibration_seconds": round(cal_s, 2), "calibration_trials": res.trials,
                             "calibration_over_budget": res.over_budget})
            print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ sweep (measurement table)
def run_sweep(args):
    """Per-configuration measurements for the results table: ms per denoising step,
    dense-equivalent and executed TFLOPS, skip fraction, % of bf16 peak; the
    fixed-threshold sweep (propagate and recompute modes, error against the dense
    tau = -inf output on the same inputs); imported random and locality masks for
    0-80% skip.
    Prints one JSON object per line.  Inputs are generated per step outside the
    timed region; each step is timed with CUDA events on its stream."""
    import dataclasses

    import torch
    from temporal_block_sparse_sm_b200 import build, liteattn, synthetic

    torch.cuda.set_device(0)
    build.build()
    liteattn.load()
    peaks, _ = load_peaks()
    bf16 = float(peaks["bf16_tflops"])
    names = args.sweep_configs.split(",")

    def trajectory(cfg, taus, mode="propagate", seed=0, dense_ref=None, import_bits=None, stride=1,
                   predicate="threshold"):
        plan = liteattn.Plan(cfg.B, cfg.H, cfg.N, cfg.d, cfg.Br, cfg.Bc, taus, pair_stride=stride, predicate=predicate)
        mask = plan.mask()
        wl = synthetic.Workload(cfg, seed=seed, device="cuda")
        o = torch.empty(wl.shape, dtype=torch.bfloat16, device="cuda")
        outs, rows = [], []
        tile_flops = 2.0 * cfg.Br * cfg.Bc * cfg.d
        dense = 4.0 * cfg.B * cfg.H * cfg.N * cfg.N * cfg.d
        for t in range(len(taus)):
            q, k, v = wl.inputs(t)
            if import_bits is not None:
                mask.import_bits(import_bits)
            elif mode == "recompute":
                mask.reset()
            torch.cuda.synchronize()
            s0 = plan.stats(mask)
            plan.timing(True)
            plan.step(q, k, v, o, mask, mask, t)
            attn_ms, step_ms, _ = plan.timing_read()
            s1 = plan.stats(mask)
            qk = s1["cum_qk_tiles"] - s0["cum_qk_tiles"]
            pv = s1["cum_pv_tiles"] - s0["cum_pv_tiles"]
            rows.append({"step": t, "tau": taus[t], "ms": step_ms, "attn_ms": attn_ms,
                         "skip": 1.0 - pv / s1["tiles_total"], "qk_skip": 1.0 - qk / s1["tiles_total"],
                         "exec_tflops": tile_flops * (qk + pv) / (attn_ms / 1e3) / 1e12,
                         "dense_eq_tflops": dense / (step_ms / 1e3) / 1e12})
            if dense_ref is not None:
                outs.append(o.clone() if t == len(taus) - 1 else None)
        plan.timing(False)
        return rows, (outs[-1] if outs else None)

    def summary(rows):
        n = len(rows)
        ms = sum(r["ms"] for r in rows) / n
        am = sum(r["attn_ms"] for r in rows)
        ex = sum(r["exec_tflops"] * r["attn_ms"] for r in rows) / am
        de = sum(r["dense_eq_tflops"] * r["ms"] for r in rows) / sum(r["ms"] for r in rows)
        return {"steps": n, "ms_per_step": ms, "dense_eq_tflops": de, "exec_tflops": ex,
                "pct_bf16_peak_exec": 100 * ex / bf16, "skip_mean": sum(r["skip"] for r in rows) / n,
                "skip_final": rows[-1]["skip"]}

    if args.sweep_policies:
        return run_policy_sweep(args, names, bf16)
    if args.sweep_calibration:
        return run_calibration_sweep(args, names, bf16)
    for name in names:
        cfg = synthetic.CONFIGS[name]
        stride = pair_stride_of(args.pair_stride, cfg)
        if name != "c5":
            rows, _ = trajectory(cfg, cfg.taus(), stride=stride)
            print(json.dumps({"sweep": "config", "workload": cfg.name, "pair_stride": stride, **summary(rows),
                              "per_step": [{k: round(v, 4) for k, v in r.items()} for r in rows]}), flush=True)
            continue
        # c5: fixed thresholds x {propagate, recompute}; error against the dense output
        _, dense_o = trajectory(cfg, [-math.inf] * cfg.T, dense_ref=True, stride=stride)
        for tau in cfg.fixed_taus:
            for mode in ("propagate", "recompute"):
                rows, o_last = trajectory(cfg, [tau] * cfg.T, mode=mode, dense_ref=True, stride=stride)
                err = (o_last.float() - dense_o.float()).abs()
                print(json.dumps({"sweep": "c5", "workload": cfg.name, "tau": tau, "mode": mode, "pair_stride": stride,
                                  **summary(rows),
                                  "err_vs_dense_max": float(err.max()), "err_vs_dense_mean": float(err.mean())}),
                      flush=True)
        # imported random masks, tau = -inf: executed throughput against the skip rate
        Tq, Tk = -(-cfg.N // cfg.Br), -(-cfg.N // cfg.Bc)
        for frac in (1.0, 0.8, 0.6, 0.4, 0.2):
            bits = synthetic.random_live_bits(cfg.B * cfg.H * Tq, Tk, frac, seed=7).numpy().astype("uint32")
            c2 = dataclasses.replace(cfg, T=3)
            rows, _ = trajectory(c2, [-math.inf] * 3, import_bits=bits, stride=stride)
            print(json.dumps({"sweep": "imported", "workload": cfg.name, "live_fraction": frac, "pair_stride": stride,
                              **summary(rows[1:])}), flush=True)
        # imported locality masks (each query tile keeps its nearest key tiles on the token grid):
        # the same skip rates with the spatio-temporal structure the pages describe; adjacent
        # query tiles per work item, and tiles one frame apart
        fstride = pair_stride_of("frame", cfg)
        for frac in (1.0, 0.8, 0.6, 0.4, 0.2):
            bits = synthetic.locality_live_bits(cfg.grid, cfg.B, cfg.H, cfg.Br, cfg.Bc, frac).numpy().astype("uint32")
            c2 = dataclasses.replace(cfg, T=3)
            for stride in (1, fstride):
                rows, _ = trajectory(c2, [-math.inf] * 3, import_bits=bits, stride=stride)
                print(json.dumps({"sweep": "imported-local", "workload": cfg.name, "live_fraction": frac,
                                  "pair_stride": stride, **summary(rows[1:])}), flush=True)
        # the fixed-recall predicate: per recall target, both modes; error against dense
        for p in (0.999, 0.99, 0.95, 0.9):
            for mode in ("propagate", "recompute"):
                rows, o_last = trajectory(cfg, [p] * cfg.T, mode=mode, dense_ref=True, predicate="recall",
                                          stride=fstride)
                err = (o_last.float() - dense_o.float()).abs()
                print(json.dumps({"sweep": "c5-recall", "workload": cfg.name, "recall": p, "mode": mode,
                                  "pair_stride": fstride, **summary(rows),
                                  "err_vs_dense_max": float(err.max()), "err_vs_dense_mean": float(err.mean())}),
                      flush=True)
    return 0


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="c4")
    ap.add_argument("--input-budget-gb", type=float, default=110.0,
                    help="device memory for per-step inputs (c4: 2.0 GB per schedule step)")
    ap.add_argument("--host-budget-gb", type=float, default=8.0,
                    help="pinned host memory for the end-to-end leg's inputs")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) leg")
    ap.add_argument("--pair-stride", default="frame",
                    help="which query tiles share a work item: adjacent (1), a stride, or 'frame' (each tile with "
                         "the one a video frame later; the default)")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="--impl reference: total oracle time of the warm-up and timed samples")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N>1: independent replicas of the workload (weak scaling, default) or one workload "
                         "with its heads split over the ranks (strong scaling)")
    ap.add_argument("--layout", default="bhnd", choices=["bhnd", "bnhd"],
                    help="tensor layout of q, k, v, o: [B,H,N,d] (default) or [B,N,H,d]")
    ap.add_argument("--sweep", action="store_true", help="print the per-configuration measurement table instead")
    ap.add_argument("--sweep-configs", default="c1,c2,c3,c4,c5")
    ap.add_argument("--sweep-policies", action="store_true",
                    help="with --sweep: compare the mask-propagation policies on each workload instead")
    ap.add_argument("--sweep-calibration", action="store_true",
                    help="with --sweep: calibrate the threshold schedule against per-step error budgets")
    ap.add_argument("--error-budget", type=float, default=5e-3,
                    help="calibration: total relative L1 error budget over the trajectory")
    ap.add_argument("--revive", type=float, default=0.02,
                    help="refresh policy: adopt the probe's mask above this divergence")
    return ap.parse_args(argv)


def main(argv=None):
    args = parse_args(argv)
    if args.sweep:
        return run_sweep(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    from temporal_block_sparse_sm_b200 import synthetic
    cfg = synthetic.CONFIGS[args.workload]
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_gpu(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
