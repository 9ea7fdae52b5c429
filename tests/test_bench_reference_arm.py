"""bench.py's reference arm (the oracle, timed on the host cores) prints one
JSON line with the contract's keys.  Runs on the CPU with a one-second step."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                          "--ref-step-budget", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600,
                         check=True).stdout
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import bench
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["config"] == bench.workload_config(__import__("block_sparse_attention_threshold_b200.synthetic",
                                                                  fromlist=["x"]).workload("refine_n32768"), 1.25, 1)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # a step is the bounded sample itself; the full-operator time is reported apart
    assert d["ms_per_step"] < 60_000 < d["extrapolated_full_operator_ms"]
    assert cb["cpu_model"]


def test_cpu_baseline_times_routing_and_dense_oracle():
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_threshold_b200 import synthetic as syn
    w = syn.workload("tiny_n1024")
    o = bench.oracle_sample_rate(w, 1.0, 0.3, dense_budget_s=0.3)
    assert o["route_s_per_head"] > 0 and o["blocks"] > 0 and o["dense_blocks"] > 0
    assert o["rate"] > 0 and o["dense_rate"] > 0
    # the extrapolation charges the routing of every head
    per_block = o["seconds"] * o["cores"] / o["blocks"]
    want = w.B * w.H * (o["route_s_per_head"] + w.M * per_block) / o["cores"]
    assert abs(o["full_s"] - want) <= 1e-9 * want


def test_library_dense_comparator_runs_or_reports_none():
    # The cuDNN SDPA backend has no CPU kernel: the helper must say so with
    # None rather than fail, and never call the timer for a backend that
    # cannot run.
    import torch
    sys.path.insert(0, ROOT)
    import bench
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    calls = []
    assert bench.library_dense_ms(q, q, q, lambda fn: calls.append(fn) or 1.0) is None
    assert calls == []
