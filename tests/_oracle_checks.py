"""Per-matrix comparison of one GPU Muon step with the fp64 oracle (numpy
only, so oracle worker processes can import it without torch).

The oracle starts from the GPU's own W_{t-1} and M_{t-1}, so every step is
checked on its own; the thresholds are the acceptance criteria:
  rel-F(O) <= 3e-2 (bf16-operand path) or 1e-4 (fp32 path),
  max |dW_gpu - dW_oracle| <= 2e-2 lr scale, scale the factor of O in Eq. 4,
  rel-F(M) <= 1e-6.
"""

from __future__ import annotations

import numpy as np

import oracle.muon_oracle as orc

TOL_O_BF16 = 3e-2
TOL_O_FP32 = 1e-4
TOL_M = 1e-6
TOL_DW = 2e-2  # times lr * scale


def rel_f(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    d = np.linalg.norm(want)
    if d == 0.0:
        return float(np.linalg.norm(got))
    return float(np.linalg.norm(got - want) / d)


def step_errors(W_prev, M_prev, G, W_new, M_new, rms_gpu, *, lr, wd, mu, ns_steps=5, coeffs=None,
                nesterov=True, scale_mode=orc.SCALE_MAX_DIM, hidden_dim=0.0) -> dict:
    """Errors of one GPU step of one matrix against the oracle (all inputs
    are the exact values the GPU saw and produced, as arrays)."""
    coeffs = orc.DEFAULT_COEFFS if coeffs is None else coeffs
    W_prev = np.asarray(W_prev, dtype=np.float64)
    R, C = W_prev.shape
    ref = orc.muon_step(W_prev, G, M_prev, lr=lr, weight_decay=wd, momentum_coef=mu, ns_steps=ns_steps,
                        coeffs=coeffs, nesterov=nesterov, scale_mode=scale_mode, hidden_dim=hidden_dim)
    if scale_mode == orc.SCALE_HIDDEN:
        scale = orc.update_scale_hidden(hidden_dim)
    elif scale_mode == orc.SCALE_UPDATE_NORM:
        scale = orc.update_norm_scale(ref.O)
    else:
        scale = orc.update_scale(R, C)
    dW_gpu = np.asarray(W_new, dtype=np.float64) - W_prev
    dW_ref = ref.W - W_prev
    out = {"dW": float(np.max(np.abs(dW_gpu - dW_ref))), "dW_bound": TOL_DW * lr * scale,
           "M": rel_f(M_new, ref.M)}
    # O recovered from the weight update: O = -(dW / lr + wd W_prev) / scale
    out["O"] = rel_f(-(dW_gpu / lr + wd * W_prev) / scale, ref.O) if scale != 0.0 else 0.0
    if rms_gpu is not None:
        out["rms"] = abs(rms_gpu - ref.rms) / ref.rms if ref.rms > 0 else abs(rms_gpu)
    return out


def assert_step_errors(out: dict, precision: str = "bf16") -> None:
    tol_o = TOL_O_FP32 if precision == "fp32" else TOL_O_BF16
    assert out["M"] <= TOL_M, out
    assert out["dW"] <= out["dW_bound"], out
    assert out["O"] <= tol_o, out
    if "rms" in out:
        assert out["rms"] <= tol_o, out


def momentum_error(M_prev, G, M_new, mu) -> float:
    """rel-F of the GPU momentum against Eq. 1, M_t = mu M_{t-1} + G_t."""
    return rel_f(M_new, orc.momentum(M_prev, G, mu))


def worker_step(args) -> dict:
    """Process-pool entry: (key, arrays, keyword arguments) -> errors."""
    key, (W_prev, M_prev, G, W_new, M_new, rms), kw = args
    out = step_errors(W_prev, M_prev, G, W_new, M_new, rms, **kw)
    out["key"] = key
    return out
