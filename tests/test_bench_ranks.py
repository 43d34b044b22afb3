"""Host logic of bench.py under several ranks, on CPU with gloo (world size 2).

The step has no exchange between GPUs, so N GPUs run N independent replicas:
the reported time is the slowest rank's, the throughput counts every rank's
work, and the reference arm runs on rank 0 only.
"""

import contextlib
import io
import json
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, ms_by_rank, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(ms_by_rank[rank], dist, "cpu")
        val = bench.replica_tflops(world, 10**12, ms)
        out.put((rank, ms, val))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value_gloo():
    world = 2
    ms_by_rank = [3.0, 5.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, ms_by_rank, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, val in res:
        assert ms == 5.0                     # the slowest replica decides
        assert val == pytest.approx(2 * 1e12 / 5e-3 / 1e12)  # both ranks' FLOPs over that time


def test_max_over_ranks_without_group_is_identity():
    assert bench.max_over_ranks(1.25) == 1.25
    assert bench.replica_tflops(1, 2 * 10**12, 1000.0) == pytest.approx(2.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]) == 0
    assert buf.getvalue() == ""


def test_reference_arm_line_on_rank_zero(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("MUON_REFERENCE_STEP_S", "0.01")
    monkeypatch.setattr(bench, "cpu_sample", lambda wl, budget, seed=0: (10**9, 0.5, 1))
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3"]) == 0
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["value"] == pytest.approx(2e9 / 1.0 / 1e12)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    for k in ("metric", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config"):
        assert k in line
    assert "workload" in line["config"]


def test_entropy_trailing_byte_count():
    # brute force: the trailing block of column j is (m-1-j) x (m-1-j) doubles
    for shape in [(1, 5), (2, 2), (7, 3), (64, 64), (2048, 1408)]:
        m = min(shape)
        want = sum(8 * (m - 1 - j) ** 2 for j in range(m - 1))
        assert bench.entropy_trailing_bytes([shape]) == want
    assert bench.entropy_trailing_bytes([(3, 4), (5, 2)]) == 8 * (4 + 1) + 8 * 1


def test_clock_sampler_keeps_the_timed_region_only():
    """Samples of nvidia-smi's CSV (timestamp first) outside the marked region
    (warm-up before it, the tail after it) are dropped; the median counts
    samples under load only; without a sampler the record says unavailable."""
    import datetime as dt
    c = bench.ClockSampler(0, interval_ms=25)
    t0 = dt.datetime(2026, 1, 2, 3, 4, 5, 0)
    c.t0, c.t1 = t0, t0 + dt.timedelta(milliseconds=300)

    def line(ms, mhz, watts, cap):
        ts = (t0 + dt.timedelta(milliseconds=ms)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, 0, {mhz}, 1965, {watts}, 0x4, Not Active, Not Active, Not Active, {cap}"

    c.lines = [line(-500, 1965, 700.0, "Not Active"),       # warm-up: dropped
               line(-10, 1900, 650.0, "Not Active"),        # within one interval of the start: kept
               line(100, 1400, 990.0, "Active"),
               line(200, 1420, 995.0, "Active"),
               line(250, 1500, 300.0, "Not Active"),        # not under load: not in the median
               line(900, 1965, 250.0, "Not Active")]        # after the region: dropped
    s = c.summary()
    assert s["samples"] == 4 and s["samples_under_load"] == 3
    assert s["sm_mhz"] == 1420.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["reason_samples"] == {"sw_power_cap": 2}
    empty = bench.ClockSampler(0)
    assert empty.summary()["reasons"] == ["unavailable"]
