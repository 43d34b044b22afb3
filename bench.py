"""Benchmark of the one-GPU Muon step on the 64+2-expert MoE batch.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload moe]

One step = one grouped muon_step over all 198 expert matrices (momentum,
Nesterov input, Frobenius normalisation, 5 quintic Newton-Schulz iterations,
weight update and the per-matrix update RMS), on synthetic inputs resident
in HBM.  Prints one JSON line (rank 0).

Metric: Newton-Schulz TFLOP/s, counted with the algorithmic (symmetry-aware)
FLOPs N (m(m+1)n + m^2(m+1) + 2 m^2 n) of every matrix with a non-zero
gradient, divided by the whole step's device time; ms per step alongside.

--gpus N under torchrun runs N independent replicas (the step has no
exchange between GPUs): value = all ranks' FLOPs / max-over-ranks time.
--impl reference times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload, in the same unit.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Newton-Schulz TFLOPS (% of B200 bf16 peak) and Muon step ms, 64-expert batch"
UNIT = "TFLOP/s"
K1_BYTES_PER_ELEM = 14          # G 2 + M 4 + 4 + hi 2 + lo 2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def ns_flops(rows: int, cols: int, steps: int) -> int:
    m, n = min(rows, cols), max(rows, cols)
    return steps * (m * (m + 1) * n + m * m * (m + 1) + 2 * m * m * n)


def ns_flops_dense(rows: int, cols: int, steps: int) -> int:
    m, n = min(rows, cols), max(rows, cols)
    return steps * (4 * m * m * n + 2 * m * m * m)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    p = os.path.join(ROOT, "matrix_orthogonalizing_optimizer_muon_b200", "csrc", "k_ns_tc.cu")
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def ncu_summary(workload: str):
    """The committed ncu summary of the GEMM kernel (per-launch DRAM bytes,
    scaled there to one launch of the workload it names, and the tensor-pipe
    utilisation per phase); None unless it was taken on the current kernel
    source and on this workload."""
    p = os.path.join(ROOT, "profiles", "ns_gemm_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_sha256_16") != kernel_source_hash() or d.get("workload") != workload:
        return None
    return d


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples of one GPU, kept for the
    timed region only.  start() launches the sampler and waits for its first
    sample (starting nvidia-smi can take longer than a short timed region);
    mark_start() and mark_end() bracket the region, and samples whose
    timestamps fall outside it (warm-up, tail) are dropped."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, interval_ms: int = 25):
        self.gpu = gpu_index
        self.interval_ms = interval_ms
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self, wait_s: float = 5.0):
        import select
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.interval_ms)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return self
        ready, _, _ = select.select([self.proc.stdout], [], [], wait_s)
        if ready:  # raw read: stop() collects the rest from the same descriptor
            self.lines += os.read(self.proc.stdout.fileno(), 1 << 16).decode(errors="replace").splitlines()
        return self

    def mark_start(self):
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        self.t1 = datetime.datetime.now()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines += out.splitlines()
            self.proc = None
        self.lines = [ln for ln in self.lines if ln.strip()]

    def in_region(self, ts: str) -> bool:
        """Whether a sample's timestamp lies in the marked region (with one
        sampling interval of slack at either end); unmarked regions and
        unparsable timestamps keep the sample."""
        if self.t0 is None or self.t1 is None:
            return True
        try:
            t = datetime.datetime.strptime(ts.strip(), "%Y/%m/%d %H:%M:%S.%f")
        except ValueError:
            return True
        slack = datetime.timedelta(milliseconds=self.interval_ms)
        return self.t0 - slack <= t <= self.t1 + slack

    def summary(self):
        """Median SM clock under load (samples with power above 400 W, the
        idle GPU draws about 200 W), the maximum clock, the throttle reasons
        seen in any sample, and how many samples showed each."""
        sm, mx, reasons = [], [], set()
        counts = {}
        loaded = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10 or not self.in_region(f[0]):
                continue
            f = f[1:]  # index, clocks, power, reasons
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            try:
                if float(f[3]) > 400.0:
                    loaded.append(float(f[1]))
            except ValueError:
                pass
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
                    counts[name] = counts.get(name, 0) + 1
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(loaded or sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "samples_under_load": len(loaded), "reason_samples": counts,
                "sm_mhz_min": min(loaded or sm), "interval_ms": self.interval_ms}


# ---------------------------------------------------------------------- replicas

def max_over_ranks(v: float, dist=None, device="cpu") -> float:
    """The largest per-rank value (the slowest replica's time); `v` itself
    without a process group."""
    if dist is None or not dist.is_initialized():
        return v
    import torch
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_tflops(world: int, flops_per_rank: int, ms_step: float) -> float:
    """Whole-job throughput of `world` independent replicas that each do
    `flops_per_rank` per step, timed by the slowest one."""
    return world * flops_per_rank / (ms_step * 1e-3) / 1e12


# ---------------------------------------------------------------------- AdamW companion leg

ADAMW_NUMELS = [65536 * 2048, 65536 * 2048] + [2048] * 16   # embedding, LM head, 16 RMSNorm gains
ADAMW_BYTES_PER_ELEM = 26                                    # P 4+4, m 4+4, v 4+4, G (bf16) 2


def bench_adamw(dev, steps: int = 20, warmup: int = 3):
    """Time the fused AdamW step on synthetic non-matrix parameters (inputs
    larger than L2); returns the bench line's `adamw_companion` object."""
    import torch
    from matrix_orthogonalizing_optimizer_muon_b200.api import AdamWPlan
    gen = torch.Generator(device=dev)
    gen.manual_seed(77)
    ts = []
    for e in ADAMW_NUMELS:
        P = torch.empty(e, device=dev).normal_(0.0, 0.02, generator=gen)
        G = torch.empty(e, device=dev).normal_(0.0, 1e-3, generator=gen).to(torch.bfloat16)
        ts.append((P, G, torch.empty(e, device=dev), torch.empty(e, device=dev)))
    plan = AdamWPlan(ADAMW_NUMELS, states=[(m, v) for _, _, m, v in ts])
    for t in range(1, warmup + 1):
        plan.step(ts, step=t, lr=4.2e-4, weight_decay=0.1)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for t in range(warmup + 1, warmup + steps + 1):
        plan.step(ts, step=t, lr=4.2e-4, weight_decay=0.1)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    plan.close()
    total = sum(ADAMW_NUMELS)
    gbs = total * ADAMW_BYTES_PER_ELEM / (ms * 1e-3) / 1e9
    peaks, kind = load_peaks()
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    return {"kernel": "adamw_kernel (fused multi-tensor AdamW)", "bound": "hbm",
            "workload": "synthetic non-matrix parameters: embedding and LM head [65536, 2048] and 16 RMSNorm "
                        "gains [2048], bf16 gradients, fp32 P/m/v",
            "elements": total, "ms_per_step": ms, "achieved": gbs, "unit": "GB/s", "peak": peak,
            "peak_source": f"hbm_gbs ({kind})", "frac": gbs / peak, "bytes_per_elem": ADAMW_BYTES_PER_ELEM}


def entropy_trailing_bytes(shapes) -> float:
    """Bytes the tridiagonal reduction streams for G0 v: the trailing
    (m-1-j) x (m-1-j) fp64 block once per column j, summed over columns."""
    total = 0.0
    for r, c in shapes:
        m = min(r, c)
        total += 8.0 * (m - 1) * m * (2 * m - 1) / 6.0
    return total


def bench_entropy(Ws, calls: int = 2):
    """Time the SVD-entropy diagnostic (Sec. 3.4) on the workload's weight
    matrices; returns the bench line's `svd_entropy` object."""
    import torch
    from matrix_orthogonalizing_optimizer_muon_b200.api import EntropyPlan
    shapes = [tuple(W.shape) for W in Ws]
    plan = EntropyPlan(shapes)
    plan_cluster = plan.cluster_size
    H = plan.compute(Ws)  # warm-up
    torch.cuda.synchronize()
    plan.profile(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(calls):
        plan.compute(Ws, H=H)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / calls
    phases = plan.profile_read()
    st, computed = plan.status()
    plan.close()
    nbytes = entropy_trailing_bytes(shapes)
    achieved = nbytes / (phases["tridiagonal"] * 1e-3) / 1e9
    peaks, kind = load_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    return {"what": "SVD entropy (Sec. 3.4) of every weight matrix after the timed steps: fp64 Gram, Householder "
                    "tridiagonal reduction, bisection on Sturm counts, entropy; one call covers all matrices",
            "matrices": len(Ws), "ms_per_call": ms, "phases_ms": phases, "status": st,
            "computed": [min(computed), max(computed)],
            "kernel": f"tridiag_kernel (fp64, {plan_cluster} CTA(s) per matrix)",
            "bound": "hbm", "achieved": achieved, "unit": "GB/s", "peak": hbm, "peak_source": f"hbm_gbs ({kind})",
            "frac": achieved / hbm,
            "achieved_basis": "the trailing block streamed once per column for G0 v (8 sum L^2 bytes per matrix) "
                              "over the whole reduction phase (panel updates and reflectors included)"}


# ---------------------------------------------------------------------- oracle (CPU) legs

def cpu_sample(wl, budget_s: float, seed: int = 0):
    """Time the fp64 oracle on whole-matrix steps of the workload until
    `budget_s` seconds have passed.  Returns (flops, seconds, matrices)."""
    import numpy as np
    import oracle.muon_oracle as orc
    from matrix_orthogonalizing_optimizer_muon_b200 import workloads as wlm
    rng = np.random.default_rng(seed)
    order = [i for i in rng.permutation(wl.n).tolist() if i not in wl.zero_grad]
    flops, spent, done = 0, 0.0, 0
    for i in order:
        _, r, c = wl.shapes[i]
        W = wlm.weight(wl, i).astype(np.float64)
        G = wlm.bf16_bits_to_f32(wlm.grad_bf16(wl, i, 0)).astype(np.float64)
        M = np.zeros_like(W)
        t0 = time.perf_counter()
        orc.muon_step(W, G, M, lr=4.2e-4, weight_decay=0.1)
        spent += time.perf_counter() - t0
        flops += ns_flops(r, c, 5)
        done += 1
        if spent >= budget_s:
            break
    return flops, spent, done


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((d.get("num_threads") or 0) for d in info) if info else (os.cpu_count() or 1)
    except Exception:
        return os.cpu_count() or 1


def blas_vendor() -> str:
    try:
        from threadpoolctl import threadpool_info
        import numpy  # noqa: F401  (loads its BLAS so threadpoolctl can see it)
        info = [d for d in threadpool_info() if d.get("user_api") == "blas"]
        return ", ".join(sorted({f"{d.get('internal_api')} {d.get('version') or ''}".strip() for d in info})) or "unknown"
    except Exception:
        return "unknown"


def torch_eager_ns_ms(Gs, zero, steps: int, abc, reps: int = 3) -> float:
    """Same-box context point, not part of the product: the quintic iteration
    written with torch.mm in bf16 (library GEMMs, no symmetry, one matrix at a
    time) over the same gradients, wide orientation.  Returns ms per pass."""
    import torch
    a, b, c = abc

    def one(G):
        X = G.t() if G.shape[0] > G.shape[1] else G
        X = (X.float() / X.float().norm()).to(torch.bfloat16)
        for _ in range(steps):
            A = X @ X.t()
            B = b * A + c * (A @ A)
            X = a * X + B @ X
        return X

    mats = [G for i, G in enumerate(Gs) if i not in zero]
    one(mats[0])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        for G in mats:
            one(G)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def library_ceiling(wl, dev, steps: int = 5, reps: int = 3):
    """Same-box context point, not part of the product: the three products of
    the quintic iteration as cuBLAS batched GEMMs (torch.bmm / baddbmm in
    bf16, dense, no symmetry) over the workload's non-zero matrices, grouped
    by shape in the wide orientation, on random inputs of the same shapes.
    Returns per-phase dense TFLOP/s and the whole iteration's rate in the
    algorithmic (symmetry-aware) count used for the kernel."""
    import torch
    groups = {}
    for i, (_, r, c) in enumerate(wl.shapes):
        if i not in wl.zero_grad:
            m, n = min(r, c), max(r, c)
            groups[(m, n)] = groups.get((m, n), 0) + 1
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    bufs = []
    for (m, n), cnt in groups.items():
        X = (torch.randn(cnt, m, n, device=dev, generator=gen) / math.sqrt(m * n)).to(torch.bfloat16)
        bufs.append((X, torch.empty(cnt, m, m, device=dev, dtype=torch.bfloat16),
                     torch.empty(cnt, m, m, device=dev, dtype=torch.bfloat16), torch.empty_like(X)))
    a, b, c = 3.4445, -4.7750, 2.0315
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    ms = [0.0, 0.0, 0.0]

    def one_pass(record):
        for _ in range(steps):
            if record:
                ev[0].record()
            for X, A, _, _ in bufs:
                torch.bmm(X, X.transpose(1, 2), out=A)
            if record:
                ev[1].record()
            for _, A, B, _ in bufs:
                torch.baddbmm(A, A, A, beta=b, alpha=c, out=B)
            if record:
                ev[2].record()
            for X, _, B, Y in bufs:
                torch.baddbmm(X, B, X, beta=a, alpha=1.0, out=Y)
            if record:
                ev[3].record()
                torch.cuda.synchronize()
                for k in range(3):
                    ms[k] += ev[k].elapsed_time(ev[k + 1])

    one_pass(False)
    torch.cuda.synchronize()
    for _ in range(reps):
        one_pass(True)
    ms = [v / reps for v in ms]
    dense = [0.0, 0.0, 0.0]
    alg = 0.0
    for (m, n), cnt in groups.items():
        dense[0] += cnt * steps * 2.0 * m * m * n
        dense[1] += cnt * steps * 2.0 * m * m * m
        dense[2] += cnt * steps * 2.0 * m * m * n
        alg += cnt * ns_flops(m, n, steps)
    del bufs
    torch.cuda.empty_cache()
    return {"what": "cuBLAS batched bf16 GEMMs (torch.bmm/baddbmm, dense, no symmetry) of the Gram, polynomial and "
                    "X-update products over the same non-zero matrices, 5 iterations; context only",
            "ms_per_step": sum(ms), "phase_ms": dict(zip(("gram", "poly", "x_update"), ms)),
            "phase_tflops_dense": {k: d / (t * 1e-3) / 1e12 for k, d, t in zip(("gram", "poly", "x_update"), dense, ms)},
            "tflops_algorithmic": alg / (sum(ms) * 1e-3) / 1e12}


def hybrid_mixed8(dev, steps: int = 5, warmup: int = 3):
    """Time the full optimizer step of the 1624-matrix mixed model: Muon over
    every matrix and AdamW over its 16 RMSNorm gains (Sec. 2.2 and Appendix D),
    one HybridStep per step on resident synthetic inputs."""
    import torch
    from matrix_orthogonalizing_optimizer_muon_b200 import workloads as wlm
    from matrix_orthogonalizing_optimizer_muon_b200.api import HybridStep
    wl = wlm.mixed8()
    shapes = [(r, c) for _, r, c in wl.shapes]
    sizes = [r * c for r, c in shapes]
    total = sum(sizes)
    gen = torch.Generator(device=dev)
    gen.manual_seed(99)
    Wbuf = torch.empty(total, device=dev).normal_(0.0, 0.02, generator=gen)
    Gbuf = torch.empty(total, device=dev).normal_(0.0, 1e-3, generator=gen).to(torch.bfloat16)
    Mbuf = torch.empty(total, device=dev)
    mats, off = [], 0
    for (r, c), e in zip(shapes, sizes):
        mats.append((Wbuf[off:off + e].view(r, c), Gbuf[off:off + e].view(r, c), Mbuf[off:off + e].view(r, c)))
        off += e
    for i in wl.zero_grad:
        mats[i][1].zero_()
    k, gsz = wl.excluded_gains, wl.gain_size
    vecs = [(torch.ones(gsz, device=dev), torch.full((gsz,), 1e-3, device=dev, dtype=torch.bfloat16),
             torch.empty(gsz, device=dev), torch.empty(gsz, device=dev)) for _ in range(k)]
    opt = HybridStep(shapes, [gsz] * k, momenta=[m for _, _, m in mats], adam_states=[(m, v) for _, _, m, v in vecs])
    ws = opt.muon.workspace_bytes
    for t in range(1, warmup + 1):
        opt.step(mats, vecs, t=t, lr=4.2e-4, weight_decay=0.1)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    opt.muon.profile(True, spans=True)
    opt.muon.profile_read()
    e0.record()
    for t in range(warmup + 1, warmup + steps + 1):
        opt.step(mats, vecs, t=t, lr=4.2e-4, weight_decay=0.1)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    prof = opt.muon.profile_read()
    st = opt.status()
    opt.close()
    nz = sum(ns_flops(r, c, 5) for i, (r, c) in enumerate(shapes) if i not in wl.zero_grad)
    gemm_ms = prof["ms"]["newton_schulz"] / max(prof["calls"], 1)
    del mats, vecs, Wbuf, Gbuf, Mbuf
    torch.cuda.empty_cache()
    return {"what": "full optimizer step of the 8-layer mixed MoE: Muon over 1624 matrices + AdamW over 16 decayed "
                    "RMSNorm gains (HybridStep), shared lr and weight decay",
            "ms_per_step": ms, "steps": steps, "status": st, "muon_workspace_gb": ws / 1e9,
            "ns_ms_per_step": gemm_ms, "ns_tflops": nz / (gemm_ms * 1e-3) / 1e12}


def other_workloads(dev, peak: float, reps: int = 10, steps: int = 10, warmup: int = 3):
    """The Newton-Schulz size sweep and the 16-layer dense stack, timed in the
    same process after the main timed region (CUDA events; Newton-Schulz time
    from the span profile).  Sweep: one plan per shape, a bf16 input of rank
    64 with singular scales decaying geometrically from 1 to 1e-3 plus noise
    (the workload recipe, drawn on the device), 5 iterations per call.  Dense
    stack: full Muon steps over its 96 matrices on resident synthetic inputs.
    Each case warms up for about 50 ms and times at least `reps` (`steps`)
    calls and about 100 ms."""
    import torch
    from matrix_orthogonalizing_optimizer_muon_b200 import workloads as wlm
    from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321)

    cur_plan = []

    def prof_on():
        cur_plan[-1].profile(True, spans=True)
        cur_plan[-1].profile_read()

    def timed(fn, n):
        # warm up for about 50 ms and time at least n calls and about 100 ms,
        # so that a short call is not timed while the clock still recovers
        # from the previous, heavier workload
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(warmup):
            fn()
        e1.record()
        torch.cuda.synchronize()
        est = max(e0.elapsed_time(e1) / warmup, 1e-3)
        for _ in range(int(50.0 / est)):
            fn()
        n = max(n, int(100.0 / est))
        torch.cuda.synchronize()
        prof_on()
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n, n

    sweep = []
    k = wlm.LOWRANK_RANK
    sig = wlm.LOWRANK_SIGMA_MIN ** (torch.arange(k, device=dev, dtype=torch.float32) / (k - 1))
    for r, c in wlm.NS_SWEEP_SHAPES:
        P = torch.randn((r, k), device=dev, generator=gen) * sig
        Q = torch.randn((c, k), device=dev, generator=gen)
        x = (P @ Q.T + wlm.LOWRANK_NOISE_STD * torch.randn((r, c), device=dev, generator=gen)).to(torch.bfloat16)
        o = torch.empty((r, c), device=dev)
        plan = MuonPlan([(r, c)])
        cur_plan.append(plan)
        ms, n = timed(lambda: plan.orthogonalize([x], [o]), reps)
        prof = plan.profile_read()
        st = plan.status()
        plan.close()
        ns_ms = prof["ms"]["newton_schulz"] / max(prof["calls"], 1)
        tf = ns_flops(r, c, 5) / (ns_ms * 1e-3) / 1e12
        sweep.append({"shape": f"{r}x{c}", "ms_per_call": ms, "calls": n, "ns_ms": ns_ms, "ns_tflops": tf,
                      "frac": tf / peak, "status": st})
        del P, Q, x, o

    wl = wlm.llama16()
    shapes = [(r, c) for _, r, c in wl.shapes]
    sizes = [r * c for r, c in shapes]
    total = sum(sizes)
    Wbuf = torch.empty(total, device=dev).normal_(0.0, 0.02, generator=gen)
    Gbuf = torch.empty(total, device=dev).normal_(0.0, 1e-3, generator=gen).to(torch.bfloat16)
    Mbuf = torch.empty(total, device=dev)
    params, off = [], 0
    for (r, c), e in zip(shapes, sizes):
        params.append((Wbuf[off:off + e].view(r, c), Gbuf[off:off + e].view(r, c), Mbuf[off:off + e].view(r, c)))
        off += e
    plan = MuonPlan(shapes, momenta=[m for _, _, m in params])
    cur_plan.append(plan)
    plan.bind(params)
    hp = dict(lr=4.2e-4, weight_decay=0.1, momentum=0.95, ns_steps=5)
    ms, n = timed(lambda: plan.step(**hp), steps)
    prof = plan.profile_read()
    st = plan.status()
    plan.close()
    ns_ms = prof["ms"]["newton_schulz"] / max(prof["calls"], 1)
    tf = sum(ns_flops(r, c, 5) for r, c in shapes) / (ns_ms * 1e-3) / 1e12
    del params, Wbuf, Gbuf, Mbuf
    torch.cuda.empty_cache()
    return {"what": "Newton-Schulz size sweep (orthogonalize, one matrix per plan) and the 16-layer dense stack "
                    "(Muon steps over 96 matrices), same process after the main timed region; frac of the same "
                    "peak as the roofline",
            "ns_sweep": sweep,
            "llama16": {"matrices": len(shapes), "ms_per_step": ms, "ns_ms_per_step": ns_ms, "ns_tflops": tf,
                        "frac": tf / peak, "steps": n, "status": st}}


def run_reference(args, wl, rank: int):
    if rank != 0:
        return
    budget = float(os.environ.get("MUON_REFERENCE_STEP_S", "2.0"))
    for _ in range(args.warmup):
        cpu_sample(wl, 0.5, seed=1)
    tot_f, tot_s, mats = 0, 0.0, 0
    for k in range(args.steps):
        f, s, d = cpu_sample(wl, budget, seed=100 + k)
        tot_f, tot_s, mats = tot_f + f, tot_s + s, mats + d
    value = tot_f / tot_s / 1e12
    sample = (f"{mats} whole-matrix oracle steps (fp64 numpy) drawn from the {wl.n}-matrix workload, "
              f"~{budget:.0f} s per timed step; FLOPs counted as for the GPU arm")
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl, args.scale),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                             "host_cpus": os.cpu_count(), "blas": blas_vendor()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


SCALE_TEXT = {"max_dim": "Eq. 4: 0.2 sqrt(max(A,B))", "hidden": "Eq. 5: 0.2 sqrt(H), H = 2048",
              "update_norm": "Eq. 6: 0.2 / RMS(O)"}


def workload_config(wl, scale: str = "max_dim"):
    nz = [s for i, s in enumerate(wl.shapes) if i not in wl.zero_grad]
    return {"workload": f"{wl.name}: {wl.n} matrices ({len(nz)} with non-zero gradient)",
            "matrices": wl.n, "elements": wl.elements, "ns_steps": 5,
            "shapes": sorted({(r, c) for _, r, c in wl.shapes}),
            "inputs": "synthetic: W ~ N(0, 0.02^2) fp32, G ~ N(0, 1e-6) bf16, M_0 = 0",
            "l2": "inputs larger than L2 (no flush needed)", "parallelism": "replicas (no exchange)",
            "update_scale": SCALE_TEXT[scale]}


# ---------------------------------------------------------------------- GPU arm

def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="moe")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-context", action="store_true", help="skip the PyTorch eager comparison point")
    ap.add_argument("--no-adamw", action="store_true", help="skip the AdamW companion measurement")
    ap.add_argument("--no-entropy", action="store_true", help="skip the SVD-entropy diagnostic measurement")
    ap.add_argument("--scale", default="max_dim", choices=["max_dim", "hidden", "update_norm"],
                    help="update scale of Sec. 3.1: Eq. 4 (default), Eq. 5 with H = 2048, Eq. 6")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--limit", type=int, default=0, help="keep only the first N matrices (small profiling case)")
    ap.add_argument("--shape", default=None,
                    help="RxC: time one matrix of this shape (with --workload ns_sweep, one of the sweep shapes)")
    ap.add_argument("--max-workspace-gb", type=float, default=0.0,
                    help="cap the plan's device memory (muon_init_ex); 0 = uncapped")
    ap.add_argument("--no-hybrid", action="store_true",
                    help="skip the hybrid Muon + AdamW step of the 1624-matrix mixed model")
    ap.add_argument("--no-ceiling", action="store_true",
                    help="skip the library batched-GEMM context point of the three product shapes")
    ap.add_argument("--no-others", action="store_true",
                    help="skip the Newton-Schulz size sweep and the 16-layer dense stack")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3

    from matrix_orthogonalizing_optimizer_muon_b200 import workloads as wlm
    wl = wlm.get(args.workload)
    if args.shape:
        r, c = (int(v) for v in args.shape.lower().split("x"))
        wl.shapes = [(f"m{r}x{c}", r, c)]
        wl.zero_grad = set()
        wl.name += f"[{r}x{c}]"
    if args.limit > 0:
        wl.shapes = wl.shapes[:args.limit]
        wl.zero_grad = {i for i in wl.zero_grad if i < args.limit}
        wl.name += f"[first {args.limit}]"
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, wl, rank)
        return 0

    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan

    dev = torch.device("cuda", local)
    shapes = [(r, c) for _, r, c in wl.shapes]
    sizes = [r * c for r, c in shapes]
    total = sum(sizes)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + rank)
    Wbuf = torch.empty(total, device=dev).normal_(0.0, 0.02, generator=gen)
    Gbuf = torch.empty(total, device=dev).normal_(0.0, 1e-3, generator=gen).to(torch.bfloat16)
    Mbuf = torch.empty(total, device=dev)
    Ws, Gs, Ms, off = [], [], [], 0
    for (r, c), e in zip(shapes, sizes):
        Ws.append(Wbuf[off:off + e].view(r, c))
        Gs.append(Gbuf[off:off + e].view(r, c))
        Ms.append(Mbuf[off:off + e].view(r, c))
        off += e
    for i in wl.zero_grad:
        Gs[i].zero_()
    cap = int(args.max_workspace_gb * 1e9)
    plan = MuonPlan(shapes, momenta=Ms, max_workspace_bytes=cap or None)
    params = list(zip(Ws, Gs, Ms))
    plan.bind(params)
    rms = torch.zeros(wl.n, device=dev)
    hp = dict(lr=4.2e-4, weight_decay=0.1, momentum=0.95, ns_steps=5, scale=args.scale, hidden_dim=2048.0)
    nz_flops = sum(ns_flops(r, c, 5) for i, (r, c) in enumerate(shapes) if i not in wl.zero_grad)
    dense_flops = sum(ns_flops_dense(r, c, 5) for i, (r, c) in enumerate(shapes) if i not in wl.zero_grad)

    def barrier():
        if dist is not None:
            dist.barrier()

    # the clock sampler runs from before the warm-up, so that its first
    # sample is in hand when the timed region starts; only samples inside the
    # region are kept
    clk = ClockSampler(local).start()
    try:
        for _ in range(args.warmup):
            plan.step(**hp, update_rms=rms)
        torch.cuda.synchronize()
    except BaseException:
        clk.stop()
        raise
    st = plan.status()
    if st != 0:
        clk.stop()
        raise RuntimeError(f"device status {st} after warm-up")

    # ---- timed region: inputs resident in HBM
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # span profile: CUDA events after the momentum pass, around each wave's
    # Newton-Schulz chain and after the update passes, none between two
    # product launches (their set-up overlaps through programmatic dependent
    # launch, which an event in between would serialise)
    plan.profile(True, spans=True)
    plan.profile_read()
    barrier()
    torch.cuda.synchronize()
    # one more event per step boundary gives the per-step times (their
    # median is reported beside the mean); a boundary event sits between two
    # steps, not inside the Newton-Schulz chain
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps - 1)]
    try:
        clk.mark_start()
        ev0.record(stream)
        for k in range(args.steps):
            plan.step(**hp, update_rms=rms)
            if k < args.steps - 1:
                step_ev[k].record(stream)
        ev1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    finally:
        clk.stop()
    bounds = [ev0] + step_ev + [ev1]
    step_ms = sorted(bounds[k].elapsed_time(bounds[k + 1]) for k in range(args.steps))
    half = len(step_ms) // 2
    ms_median = step_ms[half] if len(step_ms) % 2 else 0.5 * (step_ms[half - 1] + step_ms[half])
    barrier()
    plan.profile(False)
    prof = plan.profile_read()
    ms_step = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dist, dev)
    value = replica_tflops(world, nz_flops, ms_step)

    # ---- per-phase breakdown: a few more steps after the timed region with
    # an event after every launch (diagnostic; not part of `value`)
    diag_steps = min(args.steps, 5)
    plan.profile(True)
    plan.profile_read()
    for _ in range(diag_steps):
        plan.step(**hp, update_rms=rms)
    torch.cuda.synchronize()
    plan.profile(False)
    prof_launch = plan.profile_read()

    # ---- end to end: pinned host gradients in, update RMS out, every step.
    # Two device gradient buffers: the copy of step k+1's gradients (its own
    # stream) overlaps step k; every copy and every read-back is inside the
    # timed region, and the first copy is not hidden.
    e2e = None
    if not args.no_e2e:
        Ghost = Gbuf.cpu().pin_memory()
        rms_host = torch.empty(wl.n, dtype=torch.float32).pin_memory()
        Gbufs = [Gbuf, torch.empty_like(Gbuf)]
        views, off = [[], []], 0
        for (r, c), e in zip(shapes, sizes):
            for b in range(2):
                views[b].append(Gbufs[b][off:off + e].view(r, c))
            off += e
        pbufs = [list(zip(Ws, views[b], Ms)) for b in range(2)]
        cs = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        used = [torch.cuda.Event(), torch.cuda.Event()]

        def pipelined(nsteps):
            start = torch.cuda.Event()
            start.record(stream)
            cs.wait_event(start)
            with torch.cuda.stream(cs):
                Gbufs[0].copy_(Ghost, non_blocking=True)
                copied[0].record(cs)
            for k in range(nsteps):
                b = k % 2
                if k + 1 < nsteps:
                    with torch.cuda.stream(cs):
                        if k >= 1:
                            cs.wait_event(used[1 - b])   # step k-1 read that buffer
                        Gbufs[1 - b].copy_(Ghost, non_blocking=True)
                        copied[1 - b].record(cs)
                stream.wait_event(copied[b])
                plan.step(pbufs[b], **hp, update_rms=rms)
                used[b].record(stream)
                rms_host.copy_(rms, non_blocking=True)

        pipelined(3)
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pipelined(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist, dev)
        e2e = {"value": replica_tflops(world, nz_flops, e2e_ms), "unit": UNIT,
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": Gbuf.numel() * 2, "d2h_bytes_per_step": wl.n * 4,
               "path": "MuonPlan.step (C ABI muon_step) with each step's G copied from pinned host memory "
                       "(double-buffered: the copy of step k+1 overlaps step k) and the update RMS copied back "
                       "each step; W and M, the optimizer state, stay resident in HBM as in training"}
        del Gbufs, views, pbufs
        plan.bind(params)
    st = plan.status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timing")

    if rank != 0:
        plan.close()
        if dist is not None:
            dist.destroy_process_group()
        return 0

    peaks, peak_kind = load_peaks()
    calls = max(prof["calls"], 1)
    gemm_ms = prof["ms"]["newton_schulz"] / calls
    gemm_launches = prof["launches"]["newton_schulz"] / calls
    per_step_launches = sum(v for k, v in prof["launches"].items() if k != "newton_schulz") / calls
    dcalls = max(prof_launch["calls"], 1)
    phase_launch_ms = {k: v / dcalls for k, v in prof_launch["ms"].items()}
    achieved = nz_flops / (gemm_ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    k1_ms = prof["ms"]["momentum_normalise"] / calls
    k1_gbs = total * K1_BYTES_PER_ELEM / (k1_ms * 1e-3) / 1e9
    summary = ncu_summary(wl.name)
    traffic = summary.get("bytes_per_launch") if summary else None
    tensor_pipe = summary.get("tensor_pipe_active_pct") if summary else None

    context = None
    if not args.no_context:
        t_eager = torch_eager_ns_ms(Gs, wl.zero_grad, 5, (3.4445, -4.7750, 2.0315))
        context = {"what": "PyTorch eager Newton-Schulz (torch.mm bf16, one matrix at a time, no symmetry), "
                           "same gradients; context only",
                   "ns_ms_per_step": t_eager, "tflops_algorithmic": nz_flops / (t_eager * 1e-3) / 1e12,
                   "tflops_dense_equivalent": dense_flops / (t_eager * 1e-3) / 1e12}

    ceiling = None
    if not args.no_ceiling:
        ceiling = library_ceiling(wl, dev)

    entropy = None
    if not args.no_entropy:
        entropy = bench_entropy(Ws)

    adamw = None
    hybrid = None
    others = None
    if not (args.no_adamw and args.no_hybrid and args.no_others):
        plan.close()
        del Wbuf, Gbuf, Mbuf, Ws, Gs, Ms, params
        torch.cuda.empty_cache()
        if not args.no_adamw:
            adamw = bench_adamw(dev)
        if not args.no_hybrid:
            hybrid = hybrid_mixed8(dev)
        if not args.no_others:
            others = other_workloads(dev, peak)

    cpu = None
    if world == 1 and args.cpu_budget > 0:
        f, s, d = cpu_sample(wl, args.cpu_budget)
        cpu = {"value": f / s / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{d} whole-matrix fp64 oracle steps of the workload ({s:.1f} s), same FLOP count",
               "host_cpus": os.cpu_count(), "blas": blas_vendor()}

    clocks = clk.summary()
    config = workload_config(wl, args.scale)
    if args.scale == "update_norm":
        fin_ms = prof["ms"]["finalize"] / calls
        config["update_norm_passes"] = {
            "kernels": "update_norm_kernel (RMS(O): reads hi+lo, 4 B/elem) + apply_update_kernel "
                       "(hi+lo 4 + W 8 B/elem)", "ms_per_step": fin_ms,
            "gbs": total * 16 / (fin_ms * 1e-3) / 1e9,
            "frac_of_hbm": total * 16 / (fin_ms * 1e-3) / 1e9 / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
        "ms_per_step_median": ms_median,
        "ns_ms_per_step": gemm_ms, "ns_tflops": achieved,
        "ns_pct_of_bf16_peak": 100.0 * achieved / peak,
        "ns_tflops_dense_equivalent": dense_flops / (gemm_ms * 1e-3) / 1e12,
        "phase_ms_per_step": {k: v / calls for k, v in prof["ms"].items() if k not in ("gram", "poly", "x_update")},
        "phase_ms_per_step_launch_events": dict(
            phase_launch_ms, note=f"{diag_steps} steps after the timed region with a CUDA event after every launch "
                                  "(no launch overlap); diagnostic, not part of value"),
        "roofline": {"kernel": "ns_gemm_kernel (tcgen05, all Gram/poly/X-update launches)", "bound": "tensor",
                     "launch_time_source": "CUDA events on the launching stream around each wave's Newton-Schulz "
                                           "chain inside the timed region; average launch duration = span / "
                                           "launches",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"bf16_tflops_sustained ({peak_kind})", "traffic": traffic,
                     "ncu_tensor_pipe_active_pct": tensor_pipe,
                     "algorithmic_flops_per_launch": nz_flops / gemm_launches},
        "elementwise": {"kernel": "k1_kernel (momentum, Nesterov, norm, bf16 split)", "bound": "hbm",
                        "achieved": k1_gbs, "peak": peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
                        "unit": "GB/s", "frac": k1_gbs / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
                        "bytes_per_elem": K1_BYTES_PER_ELEM},
        "cpu_baseline": cpu,
        "context_torch_eager_ns": context,
        "context_library_batched_gemm": ceiling,
        "hybrid_step_mixed8": hybrid,
        "other_workloads": others,
        "adamw_companion": adamw,
        "svd_entropy": entropy,
        "e2e": e2e,
        "gpu_launches": int(round(per_step_launches * args.steps)),
        "clocks": clocks,
        "ns_mcycles_per_step": (gemm_ms * clocks["sm_mhz"] / 1e3) if clocks.get("sm_mhz") else None,
    }
    print(json.dumps(line), flush=True)
    plan.close()
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
