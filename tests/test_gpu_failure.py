"""Failure detection on the GPU without a fault.

muon_inject_wait_timeout makes the next call's first Newton-Schulz launch
wait, with a limit of a few microseconds, on a barrier that nothing arrives
at, before it issues any load or tensor-core instruction.  The bounded wait
runs out, the launch reports MUON_ERR_TIMEOUT through the plan's status, and
the context stays usable: the next normal step on the same plan matches the
fp64 oracle.
"""

import numpy as np
import pytest
import torch

from matrix_orthogonalizing_optimizer_muon_b200 import _lib as L
from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan

from _gpu import ABC32, LR, MU, WD, check_step, host64

pytestmark = pytest.mark.gpu

SHAPES = [(2048, 1408), (1408, 2048), (300, 520), (64, 640)]


def _step(plan, Ws, Gs, Ms, rms):
    plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32, update_rms=rms)


@pytest.mark.parametrize("wait_ns", [2000, 50000])
def test_timed_out_wait_is_reported_and_the_plan_recovers(wait_ns):
    g = torch.Generator(device="cuda")
    g.manual_seed(31)
    Ws = [torch.randn(s, device="cuda", generator=g) * 0.02 for s in SHAPES]
    Gs = [(torch.randn(s, device="cuda", generator=g) * 1e-3).to(torch.bfloat16) for s in SHAPES]
    Ms = [torch.zeros(s, device="cuda") for s in SHAPES]
    plan = MuonPlan(SHAPES)
    rms = torch.zeros(len(SHAPES), device="cuda")
    _step(plan, Ws, Gs, Ms, rms)
    assert plan.status() == L.MUON_OK
    saved = [(w.clone(), m.clone()) for w, m in zip(Ws, Ms)]

    L.muon_inject_wait_timeout(plan._plan, wait_ns)
    _step(plan, Ws, Gs, Ms, rms)
    torch.cuda.synchronize()
    assert plan.status() == L.MUON_ERR_TIMEOUT
    assert plan.status() == L.MUON_OK  # read-and-clear

    # the timed-out call's results are invalid: restore the state and step again
    for (w, m), (w0, m0) in zip(zip(Ws, Ms), saved):
        w.copy_(w0)
        m.copy_(m0)
    before = [(host64(w), host64(m), host64(gr)) for w, m, gr in zip(Ws, Ms, Gs)]
    _step(plan, Ws, Gs, Ms, rms)
    torch.cuda.synchronize()
    assert plan.status() == L.MUON_OK
    for i in range(len(SHAPES)):
        W0, M0, G0 = before[i]
        check_step(W0, M0, G0, host64(Ws[i]), host64(Ms[i]), float(rms[i]), lr=LR, wd=WD, mu=MU)
    plan.close()


def test_injection_arguments_are_checked():
    plan = MuonPlan([(64, 64)])
    for bad in (0, 1000000001):
        with pytest.raises(L.MuonError) as e:
            L.muon_inject_wait_timeout(plan._plan, bad)
        assert e.value.status == L.MUON_ERR_INVALID_ARG
    with pytest.raises(L.MuonError):
        L.muon_inject_wait_timeout(None, 1000)
    plan.close()
