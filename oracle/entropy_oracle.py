"""Plain fp64 CPU oracle for the SVD-entropy diagnostic.

TEST INFRASTRUCTURE ONLY, under the same rules as ``muon_oracle``: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import
it, and it shares no code with the CUDA path.

"Muon is Scalable for LLM Training" (Moonlight technical report, Liu et al.
2025), Sec. 3.4 "Dynamics of singular spectrum" and Fig. 4, measures how
evenly a weight matrix spreads its energy over its singular directions.  For
singular values sigma_1 .. sigma_n the SVD entropy is the Shannon entropy of
the normalised energies p_i = sigma_i^2 / sum_j sigma_j^2, divided by log n
so that it lies in [0, 1]:

    H(sigma) = -(1 / log n) sum_i p_i log p_i

Readings:
- n is the number of singular values, min(rows, cols).
- The base of the logarithm cancels; natural logs are used.
- p_i = 0 contributes 0 (the limit of p log p).
- The formula is 0 / 0 for a zero matrix (no energy) and for n = 1
  (log n = 0); both give NaN.

The singular values come from LAPACK's SVD in fp64 (a library primitive for
one step); the rest is the formula as written.
"""

from __future__ import annotations

import numpy as np


def singular_values(W) -> np.ndarray:
    """Singular values of W in fp64, descending (numpy's LAPACK SVD)."""
    W = np.asarray(W, dtype=np.float64)
    if W.ndim != 2:
        raise ValueError("W must be a matrix")
    if min(W.shape) == 0:
        return np.zeros(0)
    return np.linalg.svd(W, compute_uv=False)


def entropy_of_spectrum(sigma) -> float:
    """H(sigma) of the SVD-entropy equation (Sec. 3.4) for given singular values."""
    sigma = np.asarray(sigma, dtype=np.float64)
    n = sigma.size
    energy = sigma * sigma
    total = float(energy.sum())
    if n <= 1 or total == 0.0 or not np.isfinite(total):
        return float("nan")
    p = energy / total
    nz = p[p > 0.0]
    return float(-(nz * np.log(nz)).sum() / np.log(n))


def svd_entropy(W) -> float:
    """SVD entropy of the weight matrix W (Sec. 3.4, Fig. 4)."""
    return entropy_of_spectrum(singular_values(W))
