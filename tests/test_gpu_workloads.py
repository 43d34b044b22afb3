"""Full-size workloads through the C ABI against the fp64 oracle.

The oracle is too slow for every matrix of the large workloads, so these
tests check a seeded sample of matrices (covering every shape class) in the
exact launch configuration the benchmark uses (all matrices in one grouped
call), and the momentum of every sampled matrix at every step.  Gradients of
the large workloads are drawn on the GPU (seeded torch generator) and the
sampled matrices are copied to the host for the oracle, so both sides see
identical values.
"""

import time

import numpy as np
import pytest
import torch

import oracle.muon_oracle as orc
from matrix_orthogonalizing_optimizer_muon_b200 import workloads as wlm
from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan

from _gpu import ABC32, LR, MU, TOL_O_BF16, WD, bf16_cuda, check_step, host64, rel_f

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


def test_llama16_ten_steps_sampled():
    """Dense 16-layer stack (96 matrices), 10 consecutive grouped steps; every
    shape class is checked at the first and last step, one matrix otherwise."""
    wl = wlm.llama16()
    by_shape = {}
    for i, (_, r, c) in enumerate(wl.shapes):
        by_shape.setdefault((r, c), i)
    all_classes = sorted(by_shape.values())
    rng = np.random.default_rng(3)

    def sample(t):
        if t in (0, wl.steps - 1):
            return all_classes
        return [int(rng.integers(wl.n))]

    worst = _run_workload(wl, wl.steps, sample)
    assert worst["O"] <= TOL_O_BF16, worst


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
