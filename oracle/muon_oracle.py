"""Plain fp64 CPU oracle for the Muon optimizer step on matrix parameters.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import or run it.  It shares no code with the CUDA
path (no kernels, headers, helpers or constant tables); the two meet only on
the seeded inputs produced by the package's ``workloads`` module, which holds
no arithmetic of the method.

Source of every step: "Muon is Scalable for LLM Training" (Moonlight
technical report, Liu et al. 2025), Section 2 ("Method").  Citations below
name that page, its section and its equation.

Everything is computed in float64 with numpy.  Each function is a direct
transcription of the definition it cites; a numpy matmul is the only library
primitive used.  Readings of points the page leaves open are stated where they
are taken:

* M_0 = 0 (Sec. 2.1, below Eq. 1).
* Nesterov form: the Newton-Schulz input is mu*M_t + G_t, with M_t = mu*M_{t-1}
  + G_t and no (1-mu) damping (Sec. 2.1, Eq. 1 and the paragraph after it).
* Orientation: the iteration runs on the wide orientation (rows <= cols); a
  tall matrix is transposed in and out.  In exact arithmetic this changes
  nothing, because X p(X^T X) = p(X X^T) X for any polynomial p.
* Zero input: X_0 = M/||M||_F is undefined for M = 0; the oracle returns O = 0
  (no epsilon anywhere), so the step reduces to pure weight decay.
* Update scale: 0.2 * sqrt(max(A, B)) with [A, B] the parameter's shape
  (Sec. 2.2, Eq. 4, the "Adjusted LR" rule of Sec. 3.1, Eq. 7); the decay term
  reads W_{t-1} (decoupled, Eq. 3).  The two alternatives Sec. 3.1 compares
  are also provided: 0.2 * sqrt(H) (Eq. 5) and 0.2 / RMS(O) (Eq. 6), the
  latter 0 for O = 0.
* Update RMS: sqrt(mean(u^2)) of the orthogonalised update u, the quantity
  Algorithm 1 ("Distributed Muon", Sec. 2.3) returns for logging.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# Quintic coefficients (a, b, c) of Eq. 2, Sec. 2.1 (inherited from Jordan et
# al. 2024); N = 5 iterations and mu = 0.95 are the Sec. 2.2 "other
# hyper-parameters" choice.
DEFAULT_COEFFS = (3.4445, -4.7750, 2.0315)
DEFAULT_NS_STEPS = 5
DEFAULT_MOMENTUM = 0.95
# Sec. 2.2, Eq. 4: the update RMS is matched to AdamW's at 0.2.
DEFAULT_RMS_SCALE = 0.2

# Ways of scaling the orthogonalised update (Sec. 3.1, "Consistent update RMS")
SCALE_MAX_DIM = 0      # 0.2 * sqrt(max(A, B))          Eq. 4 = Eq. 7 ("Adjusted LR"), the method's rule
SCALE_HIDDEN = 1       # 0.2 * sqrt(H), H hidden size    Eq. 5 ("Baseline")
SCALE_UPDATE_NORM = 2  # 0.2 / RMS(O)                    Eq. 6 ("Update Norm")


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def momentum(M_prev, G, mu: float) -> np.ndarray:
    """M_t = mu * M_{t-1} + grad L_t  (Sec. 2.1, Eq. 1, first line)."""
    return mu * _f64(M_prev) + _f64(G)


def nesterov_input(M_t, G, mu: float) -> np.ndarray:
    """Nesterov-style input mu * M_t + grad L_t fed to Newton-Schulz instead of
    M_t (Sec. 2.1, paragraph after Eq. 1)."""
    return mu * _f64(M_t) + _f64(G)


def frobenius_normalise(Y) -> tuple[np.ndarray, float]:
    """X_0 = M / ||M||_F  (Sec. 2.1, Newton-Schulz paragraph).

    Returns (X_0, ||M||_F).  For M = 0 the page's division is undefined; the
    reading taken here is X_0 = 0, which makes every later iterate 0.
    """
    Y = _f64(Y)
    f = math.sqrt(float(np.sum(Y * Y)))
    if f == 0.0:
        return np.zeros_like(Y), 0.0
    return Y / f, f


def gram(X) -> np.ndarray:
    """A = X X^T, the Gram matrix inside Eq. 2 (Sec. 2.1)."""
    X = _f64(X)
    return X @ X.T


def poly(A, b: float, c: float) -> np.ndarray:
    """B = b A + c A^2, so that Eq. 2's right-hand side is a X + B X."""
    A = _f64(A)
    return b * A + c * (A @ A)


def ns_iterate(X, B, a: float) -> np.ndarray:
    """X_k = a X_{k-1} + B X_{k-1}  with B = b A + c A^2  (Eq. 2)."""
    X = _f64(X)
    return a * X + _f64(B) @ X


def newton_schulz(Y, steps: int = DEFAULT_NS_STEPS, coeffs=DEFAULT_COEFFS) -> np.ndarray:
    """O = Newton-Schulz(Y): Frobenius normalisation, then `steps` quintic
    iterations of Eq. 2 (Sec. 2.1), run in the wide orientation.

    Each iteration is  A = X X^T;  B = b A + c A^2;  X = a X + B X.
    """
    a, b, c = (float(v) for v in coeffs)
    Y = _f64(Y)
    if Y.ndim != 2:
        raise ValueError("Newton-Schulz acts on a matrix")
    transposed = Y.shape[0] > Y.shape[1]
    X = Y.T if transposed else Y
    X, f = frobenius_normalise(X)
    if f == 0.0:
        return np.zeros_like(Y)
    for _ in range(int(steps)):
        A = gram(X)
        B = poly(A, b, c)
        X = ns_iterate(X, B, a)
    return X.T.copy() if transposed else X


def update_scale(rows: int, cols: int, rms_scale: float = DEFAULT_RMS_SCALE) -> float:
    """0.2 * sqrt(max(A, B)) for a parameter of shape [A, B] (Eq. 4 / Eq. 7)."""
    return float(rms_scale) * math.sqrt(float(max(rows, cols)))


def update_scale_hidden(hidden_dim: float, rms_scale: float = DEFAULT_RMS_SCALE) -> float:
    """0.2 * sqrt(H) with H the model's hidden dimension, the same for every
    matrix (Sec. 3.1, Eq. 5, "Baseline")."""
    if not hidden_dim > 0:
        raise ValueError("Eq. 5 needs the hidden dimension H > 0")
    return float(rms_scale) * math.sqrt(float(hidden_dim))


def update_norm_scale(O, rms_scale: float = DEFAULT_RMS_SCALE) -> float:
    """Factor that makes the update's RMS exactly 0.2: 0.2 / RMS(O) (Sec. 3.1,
    Eq. 6, "Update Norm").  Reading: for O = 0 (zero input) the factor is 0,
    so the step stays pure weight decay as in the other rules."""
    r = update_rms(O)
    return 0.0 if r == 0.0 else float(rms_scale) / r


def apply_update(W, O, lr: float, weight_decay: float, scale: float) -> np.ndarray:
    """W_t = W_{t-1} - eta_t (scale * O_t + lambda W_{t-1})  (Sec. 2.2, Eq. 4;
    with scale = 1 this is Eq. 3)."""
    W = _f64(W)
    return W - lr * (scale * _f64(O) + weight_decay * W)


def update_rms(O) -> float:
    """sqrt(mean(u^2)) of the update, Algorithm 1's logged value (Sec. 2.3)."""
    O = _f64(O)
    if O.size == 0:
        return 0.0
    return math.sqrt(float(np.mean(O * O)))


@dataclass
class StepResult:
    W: np.ndarray      # W_t
    M: np.ndarray      # M_t
    O: np.ndarray      # orthogonalised update O_t (parameter orientation)
    rms: float         # sqrt(mean(O_t^2))
    Y: np.ndarray      # the Newton-Schulz input


def muon_step(W, G, M_prev, *, lr: float, weight_decay: float, momentum_coef: float = DEFAULT_MOMENTUM,
              ns_steps: int = DEFAULT_NS_STEPS, coeffs=DEFAULT_COEFFS,
              rms_scale: float = DEFAULT_RMS_SCALE, nesterov: bool = True,
              scale_mode: int = SCALE_MAX_DIM, hidden_dim: float = 0.0) -> StepResult:
    """One Muon step for one matrix parameter (Sec. 2.1 Eq. 1 with the
    Nesterov input, Eq. 2, and the Sec. 2.2 Eq. 4 update).

    1. M_t = mu M_{t-1} + G_t
    2. Y   = mu M_t + G_t   (or Y = M_t without Nesterov, plain Eq. 1)
    3. O_t = Newton-Schulz(Y)
    4. W_t = W_{t-1} - eta (scale O_t + lambda W_{t-1}), with scale
       rms_scale sqrt(max(A,B)) (Eq. 4), rms_scale sqrt(H) (Sec. 3.1 Eq. 5)
       or rms_scale / RMS(O_t) (Sec. 3.1 Eq. 6) by `scale_mode`.
    """
    W = _f64(W)
    if W.ndim != 2:
        raise ValueError("Muon updates matrix parameters only")
    M_t = momentum(M_prev, G, momentum_coef)
    Y = nesterov_input(M_t, G, momentum_coef) if nesterov else M_t
    O = newton_schulz(Y, ns_steps, coeffs)
    if scale_mode == SCALE_MAX_DIM:
        scale = update_scale(W.shape[0], W.shape[1], rms_scale)
    elif scale_mode == SCALE_HIDDEN:
        scale = update_scale_hidden(hidden_dim, rms_scale)
    elif scale_mode == SCALE_UPDATE_NORM:
        scale = update_norm_scale(O, rms_scale)
    else:
        raise ValueError(f"unknown scale_mode {scale_mode}")
    W_t = apply_update(W, O, lr, weight_decay, scale)
    return StepResult(W=W_t, M=M_t, O=O, rms=update_rms(O), Y=Y)

