"""AdamW companion step (the optimizer the pages keep for RMSNorm gains, the
embedding and the LM head; Sec. 2.2 and Appendix D of "Muon is Scalable for
LLM Training") through the C ABI, against the fp64 oracle, element by
element, run from the GPU's own previous state at every step."""

import ctypes

import numpy as np
import pytest
import torch

import oracle.adamw_oracle as ado
from matrix_orthogonalizing_optimizer_muon_b200 import _lib as L
from matrix_orthogonalizing_optimizer_muon_b200.api import AdamWPlan

from _gpu import check_adamw

pytestmark = pytest.mark.gpu

# ragged sizes across the 65536-element chunks; one fp32 gradient; decay off on two
NUMELS = [1, 7, 1000, 2048, 65536 + 3, 300001]
DTYPES = [torch.bfloat16, torch.float32, torch.bfloat16, torch.bfloat16, torch.float32, torch.bfloat16]
DECAY = [True, True, False, True, False, True]
LR, WD, BETAS, EPS = 3e-3, 0.1, (0.9, 0.95), 1e-8
F32 = lambda x: float(np.float32(x))  # the GPU receives fp32 hyper-parameters
U = 2.0 ** -24


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _tensors(seed, misaligned=False):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    out = []
    for e, dt in zip(NUMELS, DTYPES):
        if misaligned:
            # a 4-byte offset into a larger buffer: the scalar path
            P = (torch.randn(e + 1, device="cuda", generator=g) * 0.02)[1:]
        else:
            P = torch.randn(e, device="cuda", generator=g) * 0.02
        out.append([P, torch.empty(e, device="cuda", dtype=dt), torch.zeros(e, device="cuda"),
                    torch.zeros(e, device="cuda")])
    return g, out


def _check(P0, m0, v0, G, P1, m1, v1, step, decay):
    check_adamw(P0, m0, v0, G, P1, m1, v1, step=step, lr=F32(LR), wd=F32(WD), betas=(F32(BETAS[0]), F32(BETAS[1])),
                eps=F32(EPS), decay=decay)


@pytest.mark.parametrize("misaligned", [False, True])
def test_adamw_matches_oracle_over_steps(misaligned):
    g, ts = _tensors(3 + misaligned, misaligned)
    plan = AdamWPlan(NUMELS, g_dtypes=DTYPES, states=[(m, v) for _, _, m, v in ts])
    for step in range(1, 5):
        for (P, G, m, v) in ts:
            G.copy_(torch.randn(P.numel(), device="cuda", generator=g) * 1e-3)
        before = [(host(P), host(m), host(v), host(G)) for P, G, m, v in ts]
        plan.step([tuple(t) for t in ts], step=step, lr=LR, weight_decay=WD, betas=BETAS, eps=EPS, decay=DECAY)
        torch.cuda.synchronize()
        for i, (P, G, m, v) in enumerate(ts):
            P0, m0, v0, G0 = before[i]
            _check(P0, m0, v0, G0, host(P), host(m), host(v), step, DECAY[i])
    plan.close()


def test_adamw_first_step_update_rms_is_about_one():
    # Sec. 2.2: Adam and AdamW keep an update RMS of about 1 (the first step is g / (|g| + eps))
    e = 1 << 20
    P = torch.zeros(e, device="cuda")
    G = (torch.randn(e, device="cuda") * 1e-3).to(torch.bfloat16)
    m, v = torch.zeros(e, device="cuda"), torch.zeros(e, device="cuda")
    plan = AdamWPlan([e], states=[(m, v)])
    plan.step([(P, G, m, v)], step=1, lr=1.0, weight_decay=0.0)
    torch.cuda.synchronize()
    rms = float(P.double().pow(2).mean().sqrt())
    assert abs(rms - 1.0) < 1e-2
    plan.close()


def test_adamw_bitwise_deterministic():
    outs = []
    for _ in range(2):
        g, ts = _tensors(11)
        plan = AdamWPlan(NUMELS, g_dtypes=DTYPES, states=[(m, v) for _, _, m, v in ts])
        for step in (1, 2):
            for (P, G, m, v) in ts:
                G.copy_(torch.randn(P.numel(), device="cuda", generator=g) * 1e-3)
            plan.step([tuple(t) for t in ts], step=step, lr=LR, weight_decay=WD)
        torch.cuda.synchronize()
        outs.append([x.clone() for t in ts for x in (t[0], t[2], t[3])])
        plan.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_adamw_argument_errors_leave_everything_untouched():
    lib = L.load()
    g, ts = _tensors(5)
    plan = AdamWPlan(NUMELS, g_dtypes=DTYPES, states=[(m, v) for _, _, m, v in ts])
    snap = [x.clone() for t in ts for x in (t[0], t[2], t[3])]
    arr = (L.muon_adamw_param_t * len(ts))()
    for i, (P, G, m, v) in enumerate(ts):
        arr[i].P, arr[i].G, arr[i].m, arr[i].v = P.data_ptr(), G.data_ptr(), m.data_ptr(), v.data_ptr()
        arr[i].numel, arr[i].g_dtype, arr[i].decay = NUMELS[i], L.MUON_DT_BF16 if DTYPES[i] == torch.bfloat16 \
            else L.MUON_DT_FP32, 1
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    call = lambda hp, n=len(ts): lib.muon_adamw_step(plan._plan, arr, n, ctypes.byref(hp), s)
    hp = L.muon_adamw_hparams_default()
    assert call(hp, n=2) == L.MUON_ERR_SHAPE_MISMATCH
    for field, bad in (("step", 0), ("beta1", 1.0), ("beta2", -0.1), ("eps", 0.0), ("lr", float("inf"))):
        hp = L.muon_adamw_hparams_default()
        setattr(hp, field, bad)
        assert call(hp) == L.MUON_ERR_INVALID_ARG, field
    hp = L.muon_adamw_hparams_default()
    arr[3].numel = 2047
    assert call(hp) == L.MUON_ERR_SHAPE_MISMATCH
    arr[3].numel = 2048
    arr[2].G = None
    assert call(hp) == L.MUON_ERR_INVALID_ARG
    arr[2].G = ts[2][1].data_ptr()
    arr[5].m = ts[5][0].data_ptr()   # m aliasing P
    assert call(hp) == L.MUON_ERR_ALIAS
    arr[5].m = ts[5][2].data_ptr()
    torch.cuda.synchronize()
    for a, b in zip([x for t in ts for x in (t[0], t[2], t[3])], snap):
        assert torch.equal(a, b)
    plan.close()
