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

# acceptance thresholds of the bf16-operand path and of the fp32 path, and
# the comparison with the oracle, live in the numpy-only _oracle_checks
from _oracle_checks import (TOL_DW, TOL_M, TOL_O_BF16, TOL_O_FP32, assert_step_errors, momentum_error,  # noqa: E402,F401
                            rel_f, step_errors)


def bf16_cuda(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def host32(t: torch.Tensor) -> np.ndarray:
    """fp32 copy on the host (exact for bf16 and fp32 tensors)."""
    return t.detach().float().cpu().numpy()


def random_bf16(shape, seed, scale=1.0):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * np.float32(scale)
    bits = wlm.to_bf16_bits(x)
    return bf16_cuda(bits), wlm.bf16_bits_to_f32(bits).astype(np.float64)


def check_step(W_prev, M_prev, G, W_new, M_new, rms_gpu, *, lr, wd, mu, ns_steps=5, coeffs=ABC32,
               precision="bf16", nesterov=True, scale_mode=orc.SCALE_MAX_DIM, hidden_dim=0.0):
    """Compare one GPU step of one matrix with the oracle run from the GPU's
    own W_{t-1} and M_{t-1}.  Returns a dict of the measured errors."""
    out = step_errors(W_prev, M_prev, G, W_new, M_new, rms_gpu, lr=lr, wd=wd, mu=mu, ns_steps=ns_steps,
                      coeffs=coeffs, nesterov=nesterov, scale_mode=scale_mode, hidden_dim=hidden_dim)
    assert_step_errors(out, precision)
    return out


def scale_of(shape) -> float:
    return 0.2 * math.sqrt(max(shape))


def check_adamw(P0, m0, v0, G, P1, m1, v1, *, step, lr, wd, betas, eps, decay):
    """Element-wise comparison of one GPU AdamW step with the fp64 oracle,
    with bounds derived from the fp32 arithmetic of the kernel (each moment
    is one product and one fused multiply-add; the update adds a square root,
    a division and the decayed parameter).  Arguments are fp64 host arrays;
    the hyper-parameters are the fp32 values the GPU received."""
    import oracle.adamw_oracle as ado
    U = 2.0 ** -24
    b1, b2 = betas
    r = ado.adamw_step(P0, G, m0, v0, step=step, lr=lr, weight_decay=wd, betas=(b1, b2), eps=eps, decay=decay)
    tol_m = 3 * U * (np.abs(r.m) + (1 - b1) * np.abs(G)) + 1e-38
    tol_v = 3 * U * (np.abs(r.v) + (1 - b2) * G * G) + 1e-38
    assert np.all(np.abs(m1 - r.m) <= tol_m)
    assert np.all(np.abs(v1 - r.v) <= tol_v)
    bc1, bc2 = 1 - b1 ** step, 1 - b2 ** step
    den = np.sqrt(r.v / bc2) + eps
    tol_u = tol_m / bc1 / den + np.abs(r.update) * (0.5 * tol_v / np.maximum(r.v, 1e-300) + 8 * U)
    w = wd if decay else 0.0
    tol_p = 2 * U * np.abs(r.P) + lr * (tol_u + 2 * U * (np.abs(r.update) + w * np.abs(P0)))
    err = np.abs(P1 - r.P)
    assert np.all(err <= tol_p), float(np.max(err / tol_p))
    return float(np.max(err / tol_p))
