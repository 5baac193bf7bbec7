"""bench.py's command-line contract, the parts that run without a GPU (CPU).

* `--impl reference` times the CPU oracle and prints one JSON line with the
  keys the measurement contract requires (metric, value, unit, steps, warmup,
  config.workload, cpu_baseline, e2e with zero host<->device bytes, ...).
* Under a multi-rank launch only rank 0 runs the reference arm; the others
  exit 0 without output.
* Fewer than 3 warm-up steps are refused.
* The GPU arm has no CPU fallback: without a GPU it exits non-zero and prints
  no result line.
"""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(args, env_extra=None, timeout=300):
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    env.update(env_extra or {})
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


def test_default_workload_is_the_largest_single_gpu_config():
    sys.path.insert(0, ROOT)
    import bench
    a = bench.parse_args([])
    assert a.workload == "c4" and a.gpus == 1 and a.warmup >= 3


def test_reference_arm_prints_one_complete_line():
    r = _bench(["--impl", "reference", "--workload", "c2", "--steps", "1", "--warmup", "3", "--ref-seconds", "8"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["vs_baseline"] is None and d["data"] == "synthetic"
    assert d["config"]["workload"] == "c2-N8192-H12-d128"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert "extrapolated" in cb["sample"] and cb["extrapolated"] is True
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_runs_on_rank_0_only():
    r = _bench(["--impl", "reference", "--workload", "c2", "--steps", "1", "--warmup", "3", "--ref-seconds", "8"],
               {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_fewer_than_three_warmup_steps_are_refused():
    r = _bench(["--steps", "1", "--warmup", "2"])
    assert r.returncode != 0
    assert "warmup" in (r.stderr + r.stdout)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_gpu_arm_fails_loudly_without_a_gpu():
    r = _bench(["--steps", "1", "--warmup", "3"])
    assert r.returncode != 0
    assert not any(l.lstrip().startswith("{") for l in r.stdout.splitlines()), "no result line without a GPU"


def test_pair_stride_option():
    sys.path.insert(0, ROOT)
    import bench
    from temporal_block_sparse_sm_b200 import synthetic
    C = synthetic.CONFIGS
    assert bench.pair_stride_of("frame", C["c4"]) == 45 * 80 // 128 == 28
    assert bench.pair_stride_of("frame", C["c3"]) == 30 * 52 // 128 == 12
    assert bench.pair_stride_of("frame", C["c1"]) == 1          # 64-row tiles: adjacent pairs only
    assert bench.pair_stride_of("3", C["c2"]) == 3
    assert bench.parse_args([]).pair_stride in ("1", "frame")
