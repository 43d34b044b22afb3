"""The update-scale alternatives of "Muon is Scalable for LLM Training",
Sec. 3.1 (Eq. 5: 0.2 sqrt(H) for every matrix; Eq. 6: 0.2 / RMS(O), the
"Update Norm") through the C ABI, against the fp64 oracle, on both
Newton-Schulz precisions, with N = 5 and N = 0, over several steps."""

import math

import numpy as np
import pytest
import torch

import oracle.muon_oracle as orc
from matrix_orthogonalizing_optimizer_muon_b200 import _lib as L
from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan

from _gpu import ABC32, MU, WD, check_step, host64

pytestmark = pytest.mark.gpu

SHAPES = [(256, 128), (300, 520), (520, 300), (64, 64), (17, 1000), (384, 384)]
ZERO = 3   # this matrix gets a zero gradient every step
LR = 2e-3
H = 320.0


def _make(seed, fp32_ns):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    Ws = [torch.randn(s, device="cuda", generator=g) * 0.02 for s in SHAPES]
    Ms = [torch.zeros(s, device="cuda") for s in SHAPES]
    Gs = [torch.empty(s, device="cuda", dtype=torch.bfloat16) for s in SHAPES]
    return g, Ws, Ms, Gs, MuonPlan(SHAPES, fp32_ns=fp32_ns)


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("ns_steps", [5, 0])
@pytest.mark.parametrize("mode", ["hidden", "update_norm"])
def test_scale_mode_matches_oracle(mode, ns_steps, precision):
    scale_mode = orc.SCALE_HIDDEN if mode == "hidden" else orc.SCALE_UPDATE_NORM
    g, Ws, Ms, Gs, plan = _make(40 + ns_steps, precision == "fp32")
    rms = torch.zeros(len(SHAPES), device="cuda")
    for t in range(3):
        for i, G in enumerate(Gs):
            if i == ZERO:
                G.zero_()
            else:
                G.copy_(torch.randn(SHAPES[i], device="cuda", generator=g) * 1e-3)
        before = [(host64(W), host64(M), host64(G)) for W, M, G in zip(Ws, Ms, Gs)]
        plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, ns_steps=ns_steps, coeffs=ABC32,
                  precision=precision, update_rms=rms, scale=mode, hidden_dim=H)
        torch.cuda.synchronize()
        assert plan.status() == 0
        for i in range(len(SHAPES)):
            W0, M0, G0 = before[i]
            if i == ZERO:
                # O = 0: every rule leaves pure decoupled decay
                want = W0 * (1 - np.float32(LR) * np.float32(WD))
                assert np.max(np.abs(host64(Ws[i]) - want)) <= 4 * np.finfo(np.float32).eps * np.max(np.abs(W0))
                assert float(rms[i]) == 0.0
                continue
            check_step(W0, M0, G0, host64(Ws[i]), host64(Ms[i]), float(rms[i]), lr=LR, wd=WD, mu=MU,
                       ns_steps=ns_steps, precision=precision, scale_mode=scale_mode, hidden_dim=H)
    plan.close()


def test_update_norm_update_has_rms_exactly_rms_scale():
    # Eq. 6 by construction: the applied update's RMS is 0.2 for every matrix
    g, Ws, Ms, Gs, plan = _make(77, False)
    for i, G in enumerate(Gs):
        G.copy_(torch.randn(SHAPES[i], device="cuda", generator=g) * 1e-3)
    W0 = [host64(W) for W in Ws]
    lr, wd = 1e-2, 0.0
    plan.step(list(zip(Ws, Gs, Ms)), lr=lr, weight_decay=wd, momentum=MU, coeffs=ABC32, scale="update_norm")
    torch.cuda.synchronize()
    for i in range(len(SHAPES)):
        u = (W0[i] - host64(Ws[i])) / lr
        assert abs(math.sqrt(np.mean(u * u)) - 0.2) < 2e-3, (SHAPES[i], math.sqrt(np.mean(u * u)))
    plan.close()


def test_hidden_scale_equals_default_on_square_matrices():
    # Sec. 3.1: with H = max(A, B), Eq. 5 is Eq. 4; the two runs must agree bit for bit
    shape = [(384, 384)]
    outs = []
    for mode in ("max_dim", "hidden"):
        g = torch.Generator(device="cuda")
        g.manual_seed(5)
        W = torch.randn(shape[0], device="cuda", generator=g) * 0.02
        G = (torch.randn(shape[0], device="cuda", generator=g) * 1e-3).to(torch.bfloat16)
        M = torch.zeros(shape[0], device="cuda")
        plan = MuonPlan(shape)
        plan.step([(W, G, M)], lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32, scale=mode, hidden_dim=384.0)
        torch.cuda.synchronize()
        outs.append(W.clone())
        plan.close()
    assert torch.equal(outs[0], outs[1])


def test_scale_mode_argument_errors():
    import ctypes
    lib = L.load()
    W = torch.zeros(SHAPES[0], device="cuda")
    M = torch.zeros(SHAPES[0], device="cuda")
    G = torch.zeros(SHAPES[0], device="cuda", dtype=torch.bfloat16)
    plan = MuonPlan([SHAPES[0]])
    arr = (L.muon_param_t * 1)()
    arr[0].W, arr[0].G, arr[0].M = W.data_ptr(), G.data_ptr(), M.data_ptr()
    arr[0].rows, arr[0].cols = SHAPES[0]
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for mode, hdim in ((3, 0.0), (-1, 0.0), (L.MUON_SCALE_HIDDEN, 0.0), (L.MUON_SCALE_HIDDEN, float("nan")),
                       (L.MUON_SCALE_HIDDEN, -4.0)):
        hp = L.muon_hparams_default()
        hp.scale_mode, hp.hidden_dim = mode, hdim
        assert lib.muon_step(plan._plan, arr, 1, ctypes.byref(hp), None, s) == L.MUON_ERR_INVALID_ARG
    plan.close()


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", ["max_dim", "hidden", "update_norm"])
def test_gradient_turning_zero_gives_pure_decay(mode, precision):
    # a matrix routed on one step and not on the next: its Newton-Schulz
    # buffers still hold the previous step's iterate, which must not leak
    # into the update (O = 0 for Y = 0)
    shapes = [(300, 520), (520, 300)]
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    Ws = [torch.randn(s, device="cuda", generator=g) * 0.02 for s in shapes]
    Ms = [torch.zeros(s, device="cuda") for s in shapes]
    Gs = [(torch.randn(s, device="cuda", generator=g) * 1e-3).to(torch.bfloat16) for s in shapes]
    plan = MuonPlan(shapes, fp32_ns=(precision == "fp32"))
    hp = dict(lr=LR, weight_decay=WD, momentum=0.0, coeffs=ABC32, precision=precision, scale=mode, hidden_dim=H)
    plan.step(list(zip(Ws, Gs, Ms)), **hp)
    for G, M in zip(Gs, Ms):
        G.zero_()
        M.zero_()   # mu = 0 and M = 0: Y = 0 on the next step
    W0 = [host64(W) for W in Ws]
    rms = torch.full((2,), -1.0, device="cuda")
    plan.step(list(zip(Ws, Gs, Ms)), update_rms=rms, **hp)
    torch.cuda.synchronize()
    assert plan.status() == 0
    for W, w0 in zip(Ws, W0):
        want = w0 * (1 - np.float32(LR) * np.float32(WD))
        assert np.max(np.abs(host64(W) - want)) <= 4 * np.finfo(np.float32).eps * np.max(np.abs(w0))
    assert torch.equal(rms, torch.zeros(2, device="cuda"))
    plan.close()
