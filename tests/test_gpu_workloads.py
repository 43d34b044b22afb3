"""Full-size workloads through the C ABI against the fp64 oracle.

All matrices of a workload go through one grouped call, the launch
configuration the benchmark uses.  The sweep matrices and the dense 16-layer
stack are checked in full (the stack at its first and last step, with the
momentum of every matrix at every step); the 1624-matrix mixed model, whose
full oracle step takes minutes on the host, is checked on every shape class
at its first and last step and on a seeded matrix in between.  Gradients of
the large workloads are drawn on the GPU (seeded torch generator) and copied
to the host for the oracle, so both sides see identical values.
"""

import time

import numpy as np
import pytest
import torch

import oracle.muon_oracle as orc
from matrix_orthogonalizing_optimizer_muon_b200 import workloads as wlm
from matrix_orthogonalizing_optimizer_muon_b200.api import HybridStep, MuonPlan

from _gpu import (ABC32, LR, MU, TOL_M, TOL_O_BF16, WD, assert_step_errors, bf16_cuda, check_adamw, check_step, f32,
                  host32, host64, momentum_error, rel_f)
from _oracle_pool import OraclePool

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", wlm.NS_SWEEP_SHAPES)
def test_ns_sweep_full_size(shape):
    """Single-matrix Newton-Schulz sweep on the low-rank-plus-noise inputs."""
    wl = wlm.ns_sweep()
    idx = wlm.NS_SWEEP_SHAPES.index(shape)
    bits = wlm.lowrank_ns_input(wl, idx)
    x = bf16_cuda(bits)
    out = torch.empty(shape, device="cuda")
    plan = MuonPlan([shape])
    plan.orthogonalize([x], [out], ns_steps=5, coeffs=ABC32)
    torch.cuda.synchronize()
    assert plan.status() == 0
    want = orc.newton_schulz(wlm.bf16_bits_to_f32(bits).astype(np.float64), 5, ABC32)
    err = rel_f(host64(out), want)
    assert err <= TOL_O_BF16, (shape, err)
    plan.close()


def _run_workload(wl, steps, sample_fn, seed=11):
    shapes = [(r, c) for _, r, c in wl.shapes]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    Ws = [torch.empty(s, device="cuda").normal_(0.0, wlm.W_STD, generator=gen) for s in shapes]
    Ms = [torch.empty(s, device="cuda") for s in shapes]
    Gs = [torch.empty(s, device="cuda", dtype=torch.bfloat16) for s in shapes]
    plan = MuonPlan(shapes, momenta=Ms)
    rms = torch.zeros(len(shapes), device="cuda")
    worst = {"dW_frac": 0.0, "M": 0.0, "O": 0.0}
    for t in range(steps):
        for i, G in enumerate(Gs):
            if i in wl.zero_grad:
                G.zero_()
            else:
                G.copy_(torch.empty(shapes[i], device="cuda").normal_(0.0, wlm.G_STD, generator=gen))
        picks = sample_fn(t)
        before = {i: (host64(Ws[i]), host64(Ms[i]), host64(Gs[i])) for i in picks}
        plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32, update_rms=rms)
        torch.cuda.synchronize()
        assert plan.status() == 0
        for i in picks:
            W0, M0, G0 = before[i]
            e = check_step(W0, M0, G0, host64(Ws[i]), host64(Ms[i]), float(rms[i]), lr=LR, wd=WD, mu=MU)
            worst["dW_frac"] = max(worst["dW_frac"], e["dW"] / e["dW_bound"])
            worst["M"] = max(worst["M"], e["M"])
            worst["O"] = max(worst["O"], e["O"])
    plan.close()
    return worst


def test_llama16_ten_steps_every_matrix():
    """Dense 16-layer stack (96 matrices), 10 consecutive grouped steps: the
    momentum of every matrix at every step against Eq. 1, and the whole step
    (W, M, O, update RMS) of every matrix at the first and the last step,
    plus one seeded matrix at each step in between, against the oracle.  The
    oracle runs in worker processes while the GPU takes the next steps."""
    wl = wlm.llama16()
    shapes = [(r, c) for _, r, c in wl.shapes]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    Ws = [torch.empty(s, device="cuda").normal_(0.0, wlm.W_STD, generator=gen) for s in shapes]
    Ms = [torch.empty(s, device="cuda") for s in shapes]
    Gs = [torch.empty(s, device="cuda", dtype=torch.bfloat16) for s in shapes]
    plan = MuonPlan(shapes, momenta=Ms)
    rms = torch.zeros(wl.n, device="cuda")
    rng = np.random.default_rng(3)
    worst_m = 0.0
    full_steps = (0, wl.steps - 1)
    with OraclePool() as pool:
        for t in range(wl.steps):
            for i, G in enumerate(Gs):
                G.copy_(torch.empty(shapes[i], device="cuda").normal_(0.0, wlm.G_STD, generator=gen))
            picks = range(wl.n) if t in full_steps else [int(rng.integers(wl.n))]
            W_prev = {i: Ws[i].clone() for i in picks}
            M_prev = [m.clone() for m in Ms]
            plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32, update_rms=rms)
            torch.cuda.synchronize()
            assert plan.status() == 0
            rms_h = rms.cpu().numpy()
            for i in picks:
                pool.submit_step((t, i), host32(W_prev[i]), host32(M_prev[i]), host32(Gs[i]), host32(Ws[i]),
                                 host32(Ms[i]), float(rms_h[i]), lr=LR, wd=WD, mu=MU, coeffs=ABC32)
            for i in range(wl.n):
                e = momentum_error(host64(M_prev[i]), host64(Gs[i]), host64(Ms[i]), MU)
                worst_m = max(worst_m, e)
                assert e <= TOL_M, (t, i, e)
            del W_prev, M_prev
        res = pool.drain()
    assert len(res) == 2 * wl.n + wl.steps - 2
    for r in res:
        assert_step_errors(r)
    print("llama16 worst", {"O": max(r["O"] for r in res), "dW/bound": max(r["dW"] / r["dW_bound"] for r in res),
                            "M": worst_m, "rms": max(r["rms"] for r in res)})
    plan.close()


def test_mixed8_twenty_steps_sampled():
    """Mixed-shape 8-layer MoE (1624 matrices incl. routers [2048, 64] and
    low-rank KV projections), 20 grouped steps; the 16 RMSNorm gains are not
    part of the step and must stay bit-identical."""
    wl = wlm.mixed8()
    by_shape = {}
    for i, (_, r, c) in enumerate(wl.shapes):
        by_shape.setdefault((r, c), i)
    classes = sorted(by_shape.values())
    rng = np.random.default_rng(5)
    gains = torch.from_numpy(wlm.gains(wl)).cuda()
    gains_before = gains.clone()

    def sample(t):
        if t in (0, wl.steps - 1):
            return classes
        return [int(rng.integers(wl.n))]

    t0 = time.time()
    worst = _run_workload(wl, wl.steps, sample)
    assert worst["O"] <= TOL_O_BF16, worst
    assert torch.equal(gains, gains_before)
    assert time.time() - t0 < 900


def test_mixed8_hybrid_muon_and_adamw_steps():
    """The full optimizer step of the mixed model (Sec. 2.2, "Matching update
    RMS of AdamW"; Appendix D): Muon over the 1624 matrices and AdamW over
    the 16 RMSNorm gains, with weight decay, sharing lr and weight decay, in
    one HybridStep per step for 3 steps.  Every gain element is checked
    against the AdamW oracle at every step; the Muon part on every shape
    class at the first and last step and on a seeded matrix in between."""
    wl = wlm.mixed8()
    shapes = [(r, c) for _, r, c in wl.shapes]
    steps = 3
    gen = torch.Generator(device="cuda")
    gen.manual_seed(13)
    Ws = [torch.empty(s, device="cuda").normal_(0.0, wlm.W_STD, generator=gen) for s in shapes]
    Ms = [torch.empty(s, device="cuda") for s in shapes]
    Gs = [torch.empty(s, device="cuda", dtype=torch.bfloat16) for s in shapes]
    gains = torch.from_numpy(wlm.gains(wl)).cuda()
    P = [gains[k] for k in range(wl.excluded_gains)]
    Pg = [torch.empty(wl.gain_size, device="cuda", dtype=torch.bfloat16) for _ in P]
    am = [torch.empty(wl.gain_size, device="cuda") for _ in P]
    av = [torch.empty(wl.gain_size, device="cuda") for _ in P]
    opt = HybridStep(shapes, [wl.gain_size] * len(P), momenta=Ms, adam_states=list(zip(am, av)))
    by_shape = {}
    for i, s in enumerate(shapes):
        by_shape.setdefault(s, i)
    classes = sorted(by_shape.values())
    rng = np.random.default_rng(17)
    rms = torch.zeros(wl.n, device="cuda")
    worst = {"O": 0.0, "adamw": 0.0}
    for t in range(1, steps + 1):
        for i, G in enumerate(Gs):
            if i in wl.zero_grad:
                G.zero_()
            else:
                G.copy_(torch.empty(shapes[i], device="cuda").normal_(0.0, wlm.G_STD, generator=gen))
        for g in Pg:
            g.copy_(torch.empty(wl.gain_size, device="cuda").normal_(0.0, 1e-3, generator=gen))
        picks = classes if t in (1, steps) else [int(rng.integers(wl.n))]
        before = {i: (host64(Ws[i]), host64(Ms[i]), host64(Gs[i])) for i in picks}
        before_v = [(host64(p), host64(m), host64(v), host64(g)) for p, m, v, g in zip(P, am, av, Pg)]
        opt.step(list(zip(Ws, Gs, Ms)), list(zip(P, Pg, am, av)), t=t, lr=LR, weight_decay=WD, momentum=MU,
                 coeffs=ABC32, update_rms=rms)
        torch.cuda.synchronize()
        assert opt.status() == 0
        for i in picks:
            W0, M0, G0 = before[i]
            e = check_step(W0, M0, G0, host64(Ws[i]), host64(Ms[i]), float(rms[i]), lr=LR, wd=WD, mu=MU)
            worst["O"] = max(worst["O"], e["O"])
        for k, (p, m, v, _) in enumerate(zip(P, am, av, Pg)):
            P0, m0, v0, G0 = before_v[k]
            f = check_adamw(P0, m0, v0, G0, host64(p), host64(m), host64(v), step=t, lr=LR, wd=WD,
                            betas=(f32(0.9), f32(0.95)), eps=f32(1e-8), decay=True)
            worst["adamw"] = max(worst["adamw"], f)
    # the gains did move, and by decay as well as by the normalised step
    assert not torch.equal(gains, torch.from_numpy(wlm.gains(wl)).cuda())
    print("mixed8 hybrid worst", worst)
    opt.close()
