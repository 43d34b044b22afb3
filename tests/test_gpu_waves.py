"""Plans with a workspace cap (muon_init_ex with MUON_INIT_MAX_WORKSPACE).

A capped plan runs its matrices in waves that share one workspace.  Every
matrix's arithmetic is the same whichever wave holds it, so a capped plan
must give bitwise the weights, momenta, update RMS values and Newton-Schulz
outputs of an uncapped plan on the same inputs; the first test also checks
the capped plan against the fp64 oracle.
"""

import numpy as np
import pytest
import torch

from matrix_orthogonalizing_optimizer_muon_b200 import workloads as wlm
from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan
from matrix_orthogonalizing_optimizer_muon_b200 import _lib as L

from _gpu import ABC32, LR, MU, WD, check_step, f32, host64

pytestmark = pytest.mark.gpu

# MoE expert shapes, attention/KV/router shapes of the mixed model and ragged ones
SHAPES = ([(2048, 1408), (2048, 1408), (1408, 2048)] * 4 + [(2048, 3072), (3072, 2048), (2048, 512), (512, 4096),
                                                           (2048, 64), (300, 520), (520, 300), (1, 7), (17, 1000)])
ZERO = {4, 13, 18}  # matrices whose gradient is all zero (an unrouted expert among them)


def _state(shapes, seed):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    Ws = [torch.empty(s, device="cuda").normal_(0.0, wlm.W_STD, generator=gen) for s in shapes]
    Ms = [torch.zeros(s, device="cuda") for s in shapes]
    return Ws, Ms, gen


def _grads(shapes, gen, zero):
    Gs = []
    for i, s in enumerate(shapes):
        g = torch.empty(s, device="cuda").normal_(0.0, wlm.G_STD, generator=gen).to(torch.bfloat16)
        if i in zero:
            g.zero_()
        Gs.append(g)
    return Gs


def _run(plan, Ws, Ms, grads_per_step, precision="bf16", lr=LR):
    rms = []
    for Gs in grads_per_step:
        r = torch.zeros(len(Ws), device="cuda")
        plan.step(list(zip(Ws, Gs, Ms)), lr=lr, weight_decay=WD, momentum=MU, coeffs=ABC32, update_rms=r,
                  precision=precision)
        rms.append(r)
    torch.cuda.synchronize()
    assert plan.status() == 0
    return rms


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_capped_plan_is_bitwise_the_uncapped_plan(precision):
    fp32 = precision == "fp32"
    # the fp32 path is checked with a larger learning rate, so that the fp32
    # rounding of W itself stays far below its 1e-4 criterion on O
    lr = f32(0.05) if fp32 else LR
    Ws, Ms, gen = _state(SHAPES, 21)
    steps = [_grads(SHAPES, gen, ZERO) for _ in range(2)]
    Ws2 = [w.clone() for w in Ws]
    Ms2 = [m.clone() for m in Ms]
    full = MuonPlan(SHAPES, fp32_ns=fp32)
    budget = full.workspace_bytes // 3
    capped = MuonPlan(SHAPES, fp32_ns=fp32, max_workspace_bytes=budget)
    assert full.waves == 1
    assert capped.waves >= 3
    assert capped.workspace_bytes <= budget
    W_prev = [host64(w) for w in Ws2]
    rms_full = _run(full, Ws, Ms, steps[:1], precision, lr)
    rms_cap = _run(capped, Ws2, Ms2, steps[:1], precision, lr)
    for i in range(len(SHAPES)):
        assert torch.equal(Ws[i], Ws2[i]) and torch.equal(Ms[i], Ms2[i]), i
    assert torch.equal(rms_full[0], rms_cap[0])
    # the capped step against the oracle, for every matrix of the first step
    for i, s in enumerate(SHAPES):
        check_step(W_prev[i], np.zeros(s), host64(steps[0][i]), host64(Ws2[i]), host64(Ms2[i]),
                   float(rms_cap[0][i]), lr=lr, wd=WD, mu=MU, precision=precision)
    rms_full = _run(full, Ws, Ms, steps[1:], precision, lr)
    rms_cap = _run(capped, Ws2, Ms2, steps[1:], precision, lr)
    for i in range(len(SHAPES)):
        assert torch.equal(Ws[i], Ws2[i]) and torch.equal(Ms[i], Ms2[i]), i
    assert torch.equal(rms_full[0], rms_cap[0])
    # Newton-Schulz only, same plans
    xs = [g.clone() for g in steps[1]]
    o1 = [torch.empty(s, device="cuda") for s in SHAPES]
    o2 = [torch.full(s, float("nan"), device="cuda") for s in SHAPES]
    full.orthogonalize(xs, o1, coeffs=ABC32, precision=precision)
    capped.orthogonalize(xs, o2, coeffs=ABC32, precision=precision)
    torch.cuda.synchronize()
    for a, b in zip(o1, o2):
        assert torch.equal(a, b)
    full.close()
    capped.close()


def test_profiled_capped_plan_counts_every_wave():
    Ws, Ms, gen = _state(SHAPES, 22)
    Gs = _grads(SHAPES, gen, ZERO)
    plan = MuonPlan(SHAPES, max_workspace_bytes=MuonPlan(SHAPES).workspace_bytes // 4)
    waves = plan.waves
    assert waves >= 4
    plan.profile(True)
    plan.profile_read()
    plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
    prof = plan.profile_read()
    assert prof["calls"] == 1
    assert prof["launches"]["momentum_normalise"] == waves
    assert prof["launches"]["gram"] == prof["launches"]["poly"] == prof["launches"]["x_update"] == 5 * waves
    plan.close()


def test_budget_too_small_for_the_largest_matrix_is_refused():
    with pytest.raises(L.MuonError) as e:
        MuonPlan([(2048, 3072), (64, 64)], max_workspace_bytes=1 << 20)
    assert e.value.status == L.MUON_ERR_NO_MEMORY


def test_mixed8_one_step_under_an_8gb_cap_is_bitwise_the_uncapped_step():
    """The 1624-matrix mixed model: about 41 GB of workspace uncapped, here
    under 8 GB (six or more waves), one step from the same state."""
    wl = wlm.mixed8()
    shapes = [(r, c) for _, r, c in wl.shapes]
    Ws, Ms, gen = _state(shapes, 23)
    Gs = _grads(shapes, gen, wl.zero_grad)
    cap = 8 * 10 ** 9
    capped = MuonPlan(shapes, max_workspace_bytes=cap)
    assert capped.workspace_bytes <= cap
    assert capped.waves >= 5
    Ws2 = [w.clone() for w in Ws]
    Ms2 = [m.clone() for m in Ms]
    rms_cap = _run(capped, Ws2, Ms2, [Gs])[0]
    capped.close()
    torch.cuda.empty_cache()
    full = MuonPlan(shapes)
    assert full.workspace_bytes > 5 * cap
    rms_full = _run(full, Ws, Ms, [Gs])[0]
    full.close()
    assert torch.equal(rms_full, rms_cap)
    for i in range(len(shapes)):
        assert torch.equal(Ws[i], Ws2[i]) and torch.equal(Ms[i], Ms2[i]), i
