"""Boundary behaviour of the C ABI on a real device: argument errors leave
everything untouched, device status reporting, determinism and resume."""

import ctypes

import numpy as np
import pytest
import torch

from matrix_orthogonalizing_optimizer_muon_b200 import _lib as L
from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan

from _gpu import ABC32, LR, MU, WD

pytestmark = pytest.mark.gpu

SHAPES = [(256, 128), (300, 520), (520, 300)]


def make(seed=0):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    Ws = [torch.randn(s, device="cuda", generator=g) * 0.02 for s in SHAPES]
    Gs = [(torch.randn(s, device="cuda", generator=g) * 1e-3).to(torch.bfloat16) for s in SHAPES]
    Ms = [torch.zeros(s, device="cuda") for s in SHAPES]
    return Ws, Gs, Ms


def raw_params(Ws, Gs, Ms):
    arr = (L.muon_param_t * len(Ws))()
    for i, (W, G, M) in enumerate(zip(Ws, Gs, Ms)):
        arr[i].W, arr[i].G, arr[i].M = W.data_ptr(), G.data_ptr(), M.data_ptr()
        arr[i].rows, arr[i].cols = W.shape
        arr[i].g_dtype = L.MUON_DT_BF16
    return arr


def snapshot(ts):
    return [t.clone() for t in ts]


def test_argument_errors_do_not_launch_or_modify():
    lib = L.load()
    Ws, Gs, Ms = make()
    plan = MuonPlan(SHAPES)
    hp = L.muon_hparams_default()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    w0, m0 = snapshot(Ws), snapshot(Ms)
    arr = raw_params(Ws, Gs, Ms)
    # count mismatch
    assert lib.muon_step(plan._plan, arr, 2, ctypes.byref(hp), None, s) == L.MUON_ERR_SHAPE_MISMATCH
    # shape mismatch
    arr[1].cols = 521
    assert lib.muon_step(plan._plan, arr, 3, ctypes.byref(hp), None, s) == L.MUON_ERR_SHAPE_MISMATCH
    arr[1].cols = 520
    # null pointer
    arr[2].M = None
    assert lib.muon_step(plan._plan, arr, 3, ctypes.byref(hp), None, s) == L.MUON_ERR_INVALID_ARG
    arr[2].M = Ms[2].data_ptr()
    # W of one matrix aliasing M of another
    arr[0].W = Ms[0].data_ptr()
    assert lib.muon_step(plan._plan, arr, 3, ctypes.byref(hp), None, s) == L.MUON_ERR_ALIAS
    arr[0].W = Ws[0].data_ptr()
    # bad hyper-parameters
    hp.lr = float("nan")
    assert lib.muon_step(plan._plan, arr, 3, ctypes.byref(hp), None, s) == L.MUON_ERR_INVALID_ARG
    hp.lr = 1e-3
    hp.ns_steps = 33
    assert lib.muon_step(plan._plan, arr, 3, ctypes.byref(hp), None, s) == L.MUON_ERR_INVALID_ARG
    hp.ns_steps = 5
    hp.ns_precision = L.MUON_NS_FP32  # plan built without the fp32 workspace
    assert lib.muon_step(plan._plan, arr, 3, ctypes.byref(hp), None, s) == L.MUON_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    for a, b in zip(Ws + Ms, w0 + m0):
        assert torch.equal(a, b)
    assert plan.status() == 0


def test_nonfinite_gradient_is_reported():
    Ws, Gs, Ms = make(1)
    Gs[1][3, 7] = float("nan")
    plan = MuonPlan(SHAPES)
    plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
    assert plan.status() == L.MUON_ERR_NONFINITE
    assert plan.status() == 0  # read-and-clear
    assert torch.isfinite(Ws[0]).all() and torch.isfinite(Ws[2]).all()


def test_bitwise_deterministic():
    outs = []
    for _ in range(2):
        Ws, Gs, Ms = make(2)
        plan = MuonPlan(SHAPES)
        rms = torch.zeros(3, device="cuda")
        for _ in range(2):
            plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32, update_rms=rms)
        torch.cuda.synchronize()
        outs.append([t.clone() for t in Ws + Ms] + [rms.clone()])
        plan.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_resume_equals_uninterrupted():
    # 3 steps straight vs 2 steps, state copied to the host and back, 1 step
    Ws, Gs, Ms = make(3)
    plan = MuonPlan(SHAPES)
    for _ in range(3):
        plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
    torch.cuda.synchronize()
    straight = [t.clone() for t in Ws + Ms]
    Ws, Gs, Ms = make(3)
    plan2 = MuonPlan(SHAPES)
    for _ in range(2):
        plan2.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
    torch.cuda.synchronize()
    saved = [t.cpu().numpy().copy() for t in Ws + Ms]
    plan2.close()
    Ws2 = [torch.from_numpy(a).cuda() for a in saved[:3]]
    Ms2 = [torch.from_numpy(a).cuda() for a in saved[3:]]
    plan3 = MuonPlan(SHAPES)
    plan3.step(list(zip(Ws2, Gs, Ms2)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
    torch.cuda.synchronize()
    for a, b in zip(straight, Ws2 + Ms2):
        assert torch.equal(a, b)


def test_workspace_and_profile_accounting():
    plan = MuonPlan(SHAPES)
    assert plan.workspace_bytes > 0
    Ws, Gs, Ms = make(4)
    plan.profile(True)
    plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
    prof = plan.profile_read()
    assert prof["calls"] == 1
    assert prof["launches"]["gram"] == 5 and prof["launches"]["poly"] == 5 and prof["launches"]["x_update"] == 5
    assert prof["launches"]["momentum_normalise"] == 1
    assert prof["launches"]["newton_schulz"] == 15
    assert all(v >= 0 for v in prof["ms"].values())
    ns = sum(prof["ms"][k] for k in ("gram", "poly", "x_update"))
    assert prof["ms"]["newton_schulz"] == pytest.approx(ns, rel=1e-9)
    # span mode: the product launches of the call are one span
    plan.profile(True, spans=True)
    plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
    prof = plan.profile_read()
    assert prof["calls"] == 1
    assert prof["launches"]["gram"] == 5 and prof["launches"]["newton_schulz"] == 15
    assert prof["ms"]["gram"] == prof["ms"]["poly"] == prof["ms"]["x_update"] == 0.0
    assert prof["ms"]["newton_schulz"] > 0 and prof["ms"]["momentum_normalise"] > 0 and prof["ms"]["finalize"] > 0
    with pytest.raises(L.MuonError):
        L.muon_profile_enable(plan._plan, 3)


def test_rotating_buffer_sets_use_their_own_pointers():
    # the plan keeps a few device pointer tables; six distinct (W, G, M) sets
    # in rotation (more sets than tables) must each see exactly their own
    # step, bit for bit the same as a fresh plan on that set alone
    sets = [make(100 + k) for k in range(6)]
    fresh = [make(100 + k) for k in range(6)]
    plan = MuonPlan(SHAPES)
    for _ in range(2):
        for Ws, Gs, Ms in sets:
            plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
    for Ws, Gs, Ms in fresh:
        p = MuonPlan(SHAPES)
        for _ in range(2):
            p.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
        p.close()
    torch.cuda.synchronize()
    for (W1, _, M1), (W2, _, M2) in zip(sets, fresh):
        for a, b in zip(W1 + M1, W2 + M2):
            assert torch.equal(a, b)
    plan.close()


def test_step_replays_from_a_cuda_graph():
    # After one eager call with the same tensors (which uploads the pointer
    # table), a step enqueues kernels only, so it can be captured once and
    # replayed; the replays must equal eager steps bit for bit.
    Ws, Gs, Ms = make(8)
    We, Ge, Me = make(8)
    hp = dict(lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
    eager = MuonPlan(SHAPES)
    for _ in range(4):
        eager.step(list(zip(We, Ge, Me)), **hp)
    plan = MuonPlan(SHAPES)
    plan.step(list(zip(Ws, Gs, Ms)), **hp)          # step 1, eager
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            plan.step(list(zip(Ws, Gs, Ms)), **hp)  # captured, not run
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):                               # steps 2..4
        graph.replay()
    torch.cuda.synchronize()
    assert plan.status() == 0
    for a, b in zip(Ws + Ms, We + Me):
        assert torch.equal(a, b)
    del graph
    plan.close()
    eager.close()


def test_zero_input_after_nonzero_gives_exact_zero_output():
    # the Newton-Schulz launches skip a zero matrix, so its iterate buffers
    # still hold the previous call's matrix; O must nevertheless be exactly 0
    plan = MuonPlan(SHAPES)
    g = torch.Generator(device="cuda")
    g.manual_seed(31)
    xs = [torch.randn(s, device="cuda", generator=g).to(torch.bfloat16) for s in SHAPES]
    outs = [torch.empty(s, device="cuda") for s in SHAPES]
    plan.orthogonalize(xs, outs, ns_steps=5, coeffs=ABC32)
    torch.cuda.synchronize()
    assert all(bool(o.abs().max() > 0) for o in outs)
    for x in xs:
        x.zero_()
    plan.orthogonalize(xs, outs, ns_steps=5, coeffs=ABC32)
    torch.cuda.synchronize()
    assert all(torch.equal(o, torch.zeros_like(o)) for o in outs)
    plan.close()


def test_cached_binding_does_not_skip_validation_of_a_view():
    """A binding is reused only for the same addresses, shapes, dtypes and
    contiguity: a transposed view of a square tensor at a cached address, or
    a gradient of another dtype there, is validated again and rejected."""
    s = (64, 64)
    plan = MuonPlan([s])
    W = torch.zeros(s, device="cuda")
    G = torch.zeros(s, device="cuda", dtype=torch.bfloat16)
    M = torch.zeros(s, device="cuda")
    plan.bind([(W, G, M)])
    with pytest.raises(ValueError):
        plan.bind([(W.t(), G, M)])  # same address and shape, not contiguous
    with pytest.raises(TypeError):
        plan.bind([(W, G.view(torch.float16), M)])  # same address and shape, another dtype
    plan.bind([(W, G, M)])  # the cached binding is still good
    plan.step(lr=LR, weight_decay=WD, momentum=MU)
    torch.cuda.synchronize()
    assert plan.status() == 0
