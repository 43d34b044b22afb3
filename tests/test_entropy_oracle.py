"""Pins of the SVD-entropy oracle (no GPU).

The oracle computes H(sigma) of "Muon is Scalable for LLM Training",
Sec. 3.4 (SVD-entropy equation, Fig. 4).  It is pinned to:
- closed forms: equal singular values give 1, rank 1 gives 0, and two hand
  evaluations (two and three singular values);
- the binary entropy of the two eigenvalues of W W^T, found with the
  quadratic formula;
- invariances: transpose, scale, orthogonal factors on either side;
- the degenerate cases of the readings.
Planted mistakes (energies from sigma instead of sigma^2, n = max(rows,
cols), a dropped singular value) must fail the pins.
"""

import math

import numpy as np
import pytest

import oracle.entropy_oracle as ent


def gauss(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def orthonormal_rows(m, n, seed):
    q, _ = np.linalg.qr(gauss((n, m), seed))
    return q.T  # m x n with orthonormal rows (m <= n)


# log2(25) - (9 log2 9 + 16 log2 16) / 25: the entropy in bits of (9, 16) / 25,
# which is already normalised for n = 2
H_3_4 = 0.9426831892554923
# ((1/6) ln 6 + (1/3) ln 3 + (1/2) ln 2) / ln 3 for p = (1, 2, 3) / 6
H_1_2_3 = 0.920619835714305


@pytest.mark.parametrize("shape", [(5, 9), (16, 16), (64, 2048), (3, 3)])
@pytest.mark.parametrize("transpose", [False, True])
def test_equal_singular_values_give_one(shape, transpose):
    W = 0.37 * orthonormal_rows(*shape, seed=sum(shape))
    if transpose:
        W = W.T
    assert abs(ent.svd_entropy(W) - 1.0) < 1e-12


@pytest.mark.parametrize("shape", [(7, 11), (11, 7), (2, 2)])
def test_rank_one_gives_zero(shape):
    u, v = gauss(shape[0], 1), gauss(shape[1], 2)
    assert abs(ent.svd_entropy(np.outer(u, v))) < 1e-12


def test_two_singular_values_closed_form():
    W = np.diag([3.0, 4.0])
    assert abs(ent.svd_entropy(W) - H_3_4) < 1e-15
    # zero columns add no singular value: still n = 2
    Wp = np.zeros((2, 5))
    Wp[:, :2] = W
    assert abs(ent.svd_entropy(Wp) - H_3_4) < 1e-15
    # orthogonal factors on both sides leave the spectrum unchanged
    Q = orthonormal_rows(2, 2, 5)
    R = orthonormal_rows(5, 5, 6)
    assert abs(ent.svd_entropy(Q @ Wp @ R) - H_3_4) < 1e-13


def test_three_singular_values_closed_form():
    W = np.zeros((3, 4))
    W[0, 0], W[1, 1], W[2, 2] = 1.0, math.sqrt(2.0), math.sqrt(3.0)
    assert abs(ent.svd_entropy(W) - H_1_2_3) < 1e-14
    assert abs(ent.svd_entropy(W.T) - H_1_2_3) < 1e-14


@pytest.mark.parametrize("seed", range(6))
def test_two_rows_match_binary_entropy_of_quadratic_roots(seed):
    # For 2 x k, W W^T is 2 x 2: its eigenvalues are the roots of
    # x^2 - t x + d with t the trace and d the determinant.  With
    # q = l1 / (l1 + l2), H = -(q log2 q + (1 - q) log2 (1 - q)).
    W = gauss((2, 9), 100 + seed)
    G = W @ W.T
    t, d = G[0, 0] + G[1, 1], G[0, 0] * G[1, 1] - G[0, 1] * G[1, 0]
    disc = math.sqrt(t * t - 4.0 * d)
    l1, l2 = (t + disc) / 2.0, (t - disc) / 2.0
    q = l1 / (l1 + l2)
    want = -(q * math.log2(q) + (1.0 - q) * math.log2(1.0 - q))
    assert abs(ent.svd_entropy(W) - want) < 1e-12


def test_invariances():
    W = gauss((30, 50), 7)
    h = ent.svd_entropy(W)
    assert 0.0 < h < 1.0
    assert abs(ent.svd_entropy(W.T) - h) < 1e-13
    assert abs(ent.svd_entropy(-4.5e3 * W) - h) < 1e-13
    Q, R = orthonormal_rows(30, 30, 8), orthonormal_rows(50, 50, 9)
    assert abs(ent.svd_entropy(Q @ W @ R) - h) < 1e-12


def test_spread_orders_entropy():
    # more even energies give a higher entropy
    hs = [ent.entropy_of_spectrum(np.array([1.0, r, r * r, r ** 3])) for r in (0.1, 0.5, 0.9, 1.0)]
    assert all(a < b for a, b in zip(hs, hs[1:]))
    assert abs(hs[-1] - 1.0) < 1e-15


def test_degenerate_cases_are_nan():
    assert math.isnan(ent.svd_entropy(np.zeros((4, 6))))
    assert math.isnan(ent.svd_entropy(gauss((1, 8), 3)))
    assert math.isnan(ent.svd_entropy(gauss((8, 1), 3)))
    # a zero singular value contributes nothing
    W = np.zeros((3, 3))
    W[0, 0], W[1, 1] = 3.0, 4.0
    h3 = ent.svd_entropy(W)
    assert abs(h3 - H_3_4 * math.log(2) / math.log(3)) < 1e-15


MUTANTS = {
    "energy_from_sigma": lambda s: np.sqrt(s),               # p_i from sigma_i, not sigma_i^2
    "n_is_max_dim": lambda s: np.concatenate([s, np.zeros(3)]),  # extra zero "singular values"
    "dropped_value": lambda s: s[1:],                        # one term lost
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_fail_the_pins(name, monkeypatch):
    true_sv = ent.singular_values
    monkeypatch.setattr(ent, "singular_values", lambda W: MUTANTS[name](true_sv(W)))
    W3 = np.zeros((3, 4))
    W3[0, 0], W3[1, 1], W3[2, 2] = 1.0, math.sqrt(2.0), math.sqrt(3.0)
    failures = [
        abs(ent.svd_entropy(W3) - H_1_2_3) > 1e-6,
        abs(ent.svd_entropy(0.37 * orthonormal_rows(5, 9, 14)) - 1.0) > 1e-6,
    ]
    assert any(failures)
