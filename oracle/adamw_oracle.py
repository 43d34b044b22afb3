"""Plain fp64 CPU oracle for the AdamW companion step.

TEST INFRASTRUCTURE ONLY, under the same rules as ``muon_oracle``: only
``tests/`` and ``bench.py``'s CPU legs may import it, and it shares no code
with the CUDA path.

"Muon is Scalable for LLM Training" (Moonlight technical report, Liu et al.
2025) updates the parameters that are not matrices -- RMSNorm gains, the
embedding and the LM head -- with AdamW, sharing the learning rate and the
weight decay with Muon (Sec. 2.2, "Matching update RMS of AdamW"; weight decay
on the RMSNorm gains, Appendix D, "Training stability").  The pages cite AdamW (Loshchilov and
Hutter 2019) without restating it, so this is the algorithm of that paper with
decoupled weight decay and bias correction:

    m_t = beta1 m_{t-1} + (1 - beta1) g_t
    v_t = beta2 v_{t-1} + (1 - beta2) g_t^2
    p_t = p_{t-1} - lr ( m_t / (1 - beta1^t) / (sqrt(v_t / (1 - beta2^t)) + eps)
                         + wd p_{t-1} )

Readings: beta1, beta2 and eps are not given by the pages and are inputs
(defaults 0.9, 0.95, 1e-8); m_0 = v_0 = 0, t counts from 1; a parameter can
opt out of the decay (decay = False).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

DEFAULT_BETAS = (0.9, 0.95)
DEFAULT_EPS = 1e-8


@dataclass
class AdamWResult:
    P: np.ndarray
    m: np.ndarray
    v: np.ndarray
    update: np.ndarray   # the bracket above without the decay term: m_hat / (sqrt(v_hat) + eps)


def adamw_step(P, G, m_prev, v_prev, *, step: int, lr: float, weight_decay: float,
               betas=DEFAULT_BETAS, eps: float = DEFAULT_EPS, decay: bool = True) -> AdamWResult:
    """One AdamW step of one tensor (any shape), step = t >= 1."""
    if step < 1:
        raise ValueError("the step count t starts at 1")
    b1, b2 = float(betas[0]), float(betas[1])
    P = np.asarray(P, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    m = b1 * np.asarray(m_prev, dtype=np.float64) + (1.0 - b1) * G
    v = b2 * np.asarray(v_prev, dtype=np.float64) + (1.0 - b2) * G * G
    m_hat = m / (1.0 - b1 ** step)
    v_hat = v / (1.0 - b2 ** step)
    u = m_hat / (np.sqrt(v_hat) + eps)
    wd = weight_decay if decay else 0.0
    return AdamWResult(P=P - lr * (u + wd * P), m=m, v=v, update=u)


def update_rms(u) -> float:
    u = np.asarray(u, dtype=np.float64)
    return math.sqrt(float(np.mean(u * u))) if u.size else 0.0
