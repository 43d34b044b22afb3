"""bench.py end to end on the GPU, on a small slice of the MoE batch: one run
of the benchmark as a subprocess, and the keys and internal consistency of
its JSON line (the figures themselves are the benchmark's business)."""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_on_a_slice_of_the_moe_batch():
    steps = 3
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--steps", str(steps), "--warmup", "3", "--limit", "12",
           "--cpu-budget", "1", "--no-context", "--no-adamw", "--no-hybrid", "--no-ceiling", "--no-others"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "clocks", "gpu_launches",
              "ms_per_step_median", "phase_ms_per_step", "svd_entropy", "other_workloads"):
        assert k in line, k
    assert line["n_gpus"] == 1 and line["steps"] == steps and line["dtype"] == "bf16"
    assert line["config"]["matrices"] == 12 and "l2" in line["config"]
    # value: the non-zero matrices' algorithmic FLOPs over the step time
    assert line["value"] > 0 and line["ms_per_step"] > line["ns_ms_per_step"] > 0
    # one step: k1, 15 product launches, the update pass and the RMS finalisation
    assert line["gpu_launches"] == 18 * steps
    r = line["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert abs(r["achieved"] - line["ns_tflops"]) < 1e-9
    assert r["traffic"] is None  # the committed DRAM figure belongs to the full 198-matrix workload
    e = line["e2e"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] == 12 * 4 and e["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    ent = line["svd_entropy"]
    assert ent["status"] == 0 and ent["matrices"] == 12 and ent["computed"] == [1, 1]


def test_other_workloads_leg():
    """The sweep and dense-stack leg of the default line, with one timed call each."""
    import torch
    sys.path.insert(0, ROOT)
    import bench
    out = bench.other_workloads(torch.device("cuda", 0), 1400.0, reps=1, steps=1, warmup=1)
    assert [e["shape"] for e in out["ns_sweep"]] == ["1024x1024", "2048x2048", "4096x4096", "8192x8192",
                                                      "2048x8192", "8192x2048"]
    for e in out["ns_sweep"] + [out["llama16"]]:
        assert e["status"] == 0 and 0 < e["frac"] < 1.5
    assert out["llama16"]["matrices"] == 96 and out["llama16"]["ms_per_step"] > out["llama16"]["ns_ms_per_step"] > 0
