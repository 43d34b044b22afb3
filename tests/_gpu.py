"""Shared helpers of the GPU tests (imported only by tests marked gpu)."""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle.muon_oracle as orc
from matrix_orthogonalizing_optimizer_muon_b200 import workloads as wlm

# hyper-parameters exactly as the GPU sees them (fp32), promoted to double
def f32(v: float) -> float:
    return float(np.float32(v))


ABC32 = tuple(f32(v) for v in orc.DEFAULT_COEFFS)
LR, WD, MU = f32(4.2e-4), f32(0.1), f32(0.95)

# acceptance thresholds of the bf16-operand path and of the fp32 path
TOL_O_BF16 = 3e-2
TOL_O_FP32 = 1e-4
TOL_M = 1e-6
TOL_DW = 2e-2  # times lr * 0.2 * sqrt(max(rows, cols))


def rel_f(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    d = np.linalg.norm(want)
    if d == 0.0:
        return float(np.linalg.norm(got))
    return float(np.linalg.norm(got - want) / d)


def bf16_cuda(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def random_bf16(shape, seed, scale=1.0):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * np.float32(scale)
    bits = wlm.to_bf16_bits(x)
    return bf16_cuda(bits), wlm.bf16_bits_to_f32(bits).astype(np.float64)


def check_step(W_prev, M_prev, G, W_new, M_new, rms_gpu, *, lr, wd, mu, ns_steps=5, coeffs=ABC32,
               precision="bf16", nesterov=True, scale_mode=orc.SCALE_MAX_DIM, hidden_dim=0.0):
    """Compare one GPU step of one matrix with the oracle run from the GPU's
    own W_{t-1} and M_{t-1}.  Returns a dict of the measured errors."""
    R, C = W_prev.shape
    ref = orc.muon_step(W_prev, G, M_prev, lr=lr, weight_decay=wd, momentum_coef=mu, ns_steps=ns_steps,
                        coeffs=coeffs, nesterov=nesterov, scale_mode=scale_mode, hidden_dim=hidden_dim)
    if scale_mode == orc.SCALE_HIDDEN:
        scale = orc.update_scale_hidden(hidden_dim)
    elif scale_mode == orc.SCALE_UPDATE_NORM:
        scale = orc.update_norm_scale(ref.O)
    else:
        scale = orc.update_scale(R, C)
    dW_gpu = W_new - W_prev
    dW_ref = ref.W - W_prev
    bound = TOL_DW * lr * scale
    err_dw = float(np.max(np.abs(dW_gpu - dW_ref)))
    err_m = rel_f(M_new, ref.M)
    # O recovered from the weight update: O = -(dW / lr + wd W_prev) / scale
    O_gpu = -(dW_gpu / lr + wd * W_prev) / scale
    err_o = rel_f(O_gpu, ref.O)
    out = {"dW": err_dw, "dW_bound": bound, "M": err_m, "O": err_o}
    if rms_gpu is not None:
        out["rms"] = abs(rms_gpu - ref.rms) / max(ref.rms, 1e-30) if ref.rms > 0 else abs(rms_gpu)
    tol_o = TOL_O_FP32 if precision == "fp32" else TOL_O_BF16
    assert err_m <= TOL_M, out
    assert err_dw <= bound, out
    assert err_o <= tol_o, out
    if rms_gpu is not None:
        assert out["rms"] <= tol_o, out
    return out


def scale_of(shape) -> float:
    return 0.2 * math.sqrt(max(shape))
