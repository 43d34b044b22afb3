"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own formulas: Newton-Schulz is checked
against its SVD closed form, against the textbook cubic iteration's limit (the
polar factor, also from scipy), against brute-force scalar iterations on
diagonal and rank-one inputs, and against exact invariances; the momentum and
update rules are checked against their unrolled closed forms and Lemma 1 of
"Muon is Scalable for LLM Training" (Sec. 2.2, proof in Appendix A).
The mutation tests at the end plant plausible mistakes in the oracle and check
that at least one pin catches each.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle.muon_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "printed_values.json")
ABC = orc.DEFAULT_COEFFS


def phi_n(x: float, steps: int, coeffs=ABC) -> float:
    """Scalar quintic map applied `steps` times, in plain Python."""
    a, b, c = coeffs
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def svd_closed_form(Y: np.ndarray, steps: int, coeffs=ABC) -> np.ndarray:
    """U diag(phi^N(sigma / ||Y||_F)) V^T from a thin SVD."""
    U, s, Vt = np.linalg.svd(Y, full_matrices=False)
    f = math.sqrt(float(np.sum(s * s)))
    d = np.array([phi_n(float(v) / f, steps, coeffs) for v in s])
    return (U * d[None, :]) @ Vt


def rel_f(x, y) -> float:
    return float(np.linalg.norm(x - y) / max(np.linalg.norm(y), 1e-300))


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


SHAPES = [(8, 8), (5, 12), (12, 5), (1, 7), (7, 1), (33, 64), (64, 33), (128, 256), (256, 128)]


# ------------------------------------------------------------------ Newton-Schulz pins

@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("steps", [0, 1, 2, 5])
def test_ns_equals_svd_closed_form(shape, steps):
    Y = rand(shape, 1 + shape[0] * 1000 + shape[1])
    got = orc.newton_schulz(Y, steps)
    want = svd_closed_form(Y, steps)
    assert got.shape == Y.shape
    assert rel_f(got, want) < 1e-12


def test_ns_closed_form_low_rank_plus_noise_1024():
    # the Newton-Schulz sweep's structure at a size the SVD still handles fast
    rng = np.random.default_rng(7)
    P, Q = rng.standard_normal((256, 64)), rng.standard_normal((384, 64))
    sig = 1e-3 ** (np.arange(64) / 63)
    Y = (P * sig) @ Q.T + 1e-2 * rng.standard_normal((256, 384))
    assert rel_f(orc.newton_schulz(Y, 5), svd_closed_form(Y, 5)) < 1e-11


def test_ns_rank_deficient_keeps_null_space():
    rng = np.random.default_rng(3)
    Y = rng.standard_normal((20, 3)) @ rng.standard_normal((3, 30))  # rank 3
    O = orc.newton_schulz(Y, 5)
    assert rel_f(O, svd_closed_form(Y, 5)) < 1e-11
    assert np.linalg.matrix_rank(O, tol=1e-8) == 3


@pytest.mark.parametrize("shape", [(6, 6), (6, 9), (9, 6)])
def test_textbook_cubic_iteration_reaches_polar_factor(shape):
    # (a, b, c) = (1.5, -0.5, 0) is the classical cubic Newton-Schulz iteration
    # whose fixed point is the orthogonal polar factor U V^T.
    rng = np.random.default_rng(11)
    m, n = min(shape), max(shape)
    U, _ = np.linalg.qr(rng.standard_normal((m, m)))
    V, _ = np.linalg.qr(rng.standard_normal((n, m)))
    s = np.linspace(1.0, 0.2, m)
    Y = (U * s) @ V.T
    if shape[0] > shape[1]:
        Y = Y.T
    O = orc.newton_schulz(Y, 60, (1.5, -0.5, 0.0))
    if Y.shape[0] <= Y.shape[1]:
        polar_u, _ = scipy.linalg.polar(Y.T)   # right polar of the transpose
        want = polar_u.T
    else:
        want, _ = scipy.linalg.polar(Y)
    assert np.max(np.abs(O - want)) < 1e-12


def test_ns_zero_steps_is_frobenius_normalised_input():
    Y = rand((9, 14), 5)
    assert np.max(np.abs(orc.newton_schulz(Y, 0) - Y / np.sqrt((Y * Y).sum()))) < 1e-15


def test_ns_zero_input_is_zero():
    for shape in [(4, 4), (3, 8), (8, 3)]:
        O = orc.newton_schulz(np.zeros(shape), 5)
        assert O.shape == shape and not O.any()


@pytest.mark.parametrize("shape", [(7, 11), (16, 16)])
def test_ns_diagonal_brute_force(shape):
    d = np.array([3.0, -1.0, 0.5, 2.0, 0.25, 1.5, -0.75, 1.0, 0.1, 2.5, 0.6, 0.9, 1.1, 0.3, 0.05, 4.0])
    m = min(shape)
    Y = np.zeros(shape)
    for i in range(m):
        Y[i, i] = d[i]
    f = math.sqrt(sum(d[i] ** 2 for i in range(m)))
    O = orc.newton_schulz(Y, 5)
    for i in range(shape[0]):
        for j in range(shape[1]):
            want = phi_n(d[i] / f, 5) if i == j else 0.0
            assert abs(O[i, j] - want) < 1e-13


def test_ns_rank_one_outer_product():
    rng = np.random.default_rng(2)
    u, v = rng.standard_normal(13), rng.standard_normal(5)
    O = orc.newton_schulz(np.outer(u, v), 5)
    want = phi_n(1.0, 5) * np.outer(u / np.linalg.norm(u), v / np.linalg.norm(v))
    assert np.max(np.abs(O - want)) < 1e-13


@pytest.mark.parametrize("shape", [(10, 17), (17, 10), (12, 12)])
def test_ns_transpose_equivariance(shape):
    Y = rand(shape, 21)
    assert np.max(np.abs(orc.newton_schulz(Y.T, 5) - orc.newton_schulz(Y, 5).T)) < 1e-13


def test_ns_scale_invariance_and_oddness():
    Y = rand((9, 20), 4)
    O = orc.newton_schulz(Y, 5)
    assert np.max(np.abs(orc.newton_schulz(37.5 * Y, 5) - O)) < 1e-13
    assert np.max(np.abs(orc.newton_schulz(1e-6 * Y, 5) - O)) < 1e-13
    assert np.max(np.abs(orc.newton_schulz(-Y, 5) + O)) < 1e-15


def test_ns_orthogonal_equivariance():
    rng = np.random.default_rng(8)
    Y = rng.standard_normal((10, 18))
    Q, _ = np.linalg.qr(rng.standard_normal((10, 10)))
    P, _ = np.linalg.qr(rng.standard_normal((18, 18)))
    assert np.max(np.abs(orc.newton_schulz(Q @ Y @ P, 5) - Q @ orc.newton_schulz(Y, 5) @ P)) < 1e-13


def test_ns_output_is_not_orthogonal_with_quintic_coefficients():
    # The quintic map is tuned for speed, not convergence: after 5 steps the
    # singular values sit in a band around 1 instead of at 1 (Sec. 2.1 asks
    # only for a fixed point "near 1").
    Y = rand((64, 128), 9)
    s = np.linalg.svd(orc.newton_schulz(Y, 5), compute_uv=False)
    assert 0.6 < s.min() < s.max() < 1.25
    assert s.max() - s.min() > 0.05


# ------------------------------------------------------------------ update scale (Lemma 1)

@pytest.mark.parametrize("shape", [(16, 16), (16, 64), (64, 16), (31, 7), (1, 9)])
def test_lemma1_full_rank_polar_update_rms(shape):
    Y = rand(shape, 31)
    U, _, Vt = np.linalg.svd(Y, full_matrices=False)
    O = U @ Vt                                   # exact orthogonalisation, full rank
    assert abs(orc.update_rms(O) - 1.0 / math.sqrt(max(shape))) < 1e-14
    W = rand(shape, 32)
    dW = orc.apply_update(W, O, lr=1.0, weight_decay=0.0, scale=orc.update_scale(*shape)) - W
    assert abs(orc.update_rms(dW) - 0.2) < 1e-13


@pytest.mark.parametrize("r", [1, 3, 6])
def test_lemma1_rank_r_rms(r):
    m, n = 6, 10
    rng = np.random.default_rng(r)
    U, _ = np.linalg.qr(rng.standard_normal((n, n)))
    V, _ = np.linalg.qr(rng.standard_normal((m, m)))
    X = U[:, :r] @ V[:r, :]
    assert abs(orc.update_rms(X) - math.sqrt(r / (m * n))) < 1e-14


def test_printed_values_match_oracle_defaults():
    g = json.load(open(GOLDEN))
    assert tuple(g["ns_coefficients"]["value"]) == orc.DEFAULT_COEFFS
    assert g["ns_steps"]["value"] == orc.DEFAULT_NS_STEPS
    assert g["momentum"]["value"] == orc.DEFAULT_MOMENTUM
    assert g["rms_scale"]["value"] == orc.DEFAULT_RMS_SCALE
    (r1, c1), (r2, c2) = g["mlp_vs_attention_update_ratio"]["shapes"]
    ratio = orc.update_scale(r1, c1) / orc.update_scale(r2, c2)
    assert abs(ratio - g["mlp_vs_attention_update_ratio"]["value"]) < 1e-15
    # 0.2 * sqrt(256) for the tiny [256, 128] workload
    assert abs(orc.update_scale(256, 128) - 3.2) < 1e-15
    assert orc.update_scale(128, 256) == orc.update_scale(256, 128)


# ------------------------------------------------------------------ momentum and the full step

def _run_steps(W0, Gs, **hp):
    W, M = W0, np.zeros_like(W0)
    outs = []
    for G in Gs:
        r = orc.muon_step(W, G, M, **hp)
        outs.append(r)
        W, M = r.W, r.M
    return outs


def test_momentum_unrolled_closed_form_and_nesterov_input():
    mu, T = 0.95, 6
    Gs = [rand((5, 8), 100 + t) for t in range(T)]
    outs = _run_steps(rand((5, 8), 99), Gs, lr=1e-3, weight_decay=0.1, momentum_coef=mu)
    for t in range(T):
        Mt = sum(mu ** (t - k) * Gs[k] for k in range(t + 1))    # M_0 = 0
        assert np.max(np.abs(outs[t].M - Mt)) < 1e-13
        assert np.max(np.abs(outs[t].Y - (mu * Mt + Gs[t]))) < 1e-13


def test_plain_momentum_feeds_M_t():
    Gs = [rand((4, 6), 200 + t) for t in range(3)]
    outs = _run_steps(rand((4, 6), 199), Gs, lr=1e-3, weight_decay=0.0, momentum_coef=0.9, nesterov=False)
    assert np.max(np.abs(outs[-1].Y - outs[-1].M)) == 0.0


def test_zero_gradient_is_pure_decoupled_weight_decay():
    W0 = rand((6, 9), 5)
    lr, wd = 0.01, 0.1
    outs = _run_steps(W0, [np.zeros((6, 9))] * 4, lr=lr, weight_decay=wd)
    for t, r in enumerate(outs, start=1):
        assert not r.O.any() and r.rms == 0.0
        assert np.max(np.abs(r.W - (1 - lr * wd) ** t * W0)) < 1e-15


@pytest.mark.parametrize("shape", [(12, 20), (20, 12)])
def test_full_step_against_svd_route(shape):
    # W_t = W_{t-1} - eta (0.2 sqrt(max) U phi^5(S/||Y||) V^T + lambda W_{t-1}),
    # with Y = mu M_t + G_t from the unrolled momentum; a large eta makes the
    # ordering of decay and update visible.
    mu, lr, wd = 0.95, 0.5, 0.3
    Gs = [rand(shape, 300 + t) for t in range(3)]
    W0 = rand(shape, 299)
    outs = _run_steps(W0, Gs, lr=lr, weight_decay=wd, momentum_coef=mu)
    W = W0
    for t in range(3):
        Mt = sum(mu ** (t - k) * Gs[k] for k in range(t + 1))
        O = svd_closed_form(mu * Mt + Gs[t], 5)
        W = W - lr * (0.2 * math.sqrt(max(shape)) * O + wd * W)
        assert np.max(np.abs(outs[t].W - W)) < 1e-12 * max(1.0, np.max(np.abs(W)))
        assert abs(outs[t].rms - math.sqrt(np.mean(O * O))) < 1e-13


# ------------------------------------------------------------------ update-scale alternatives (Sec. 3.1)

def _one_step(shape, seed, **hp):
    W0 = rand(shape, seed)
    G = rand(shape, seed + 1)
    return W0, orc.muon_step(W0, G, np.zeros(shape), **hp)


def _update_part(W0, r, lr, wd):
    """u with W_t = W_{t-1} - lr (u + wd W_{t-1})."""
    return (W0 * (1 - lr * wd) - r.W) / lr


def test_hidden_dim_scale_matches_eq4_on_square_and_printed_ratio():
    # Sec. 3.1: for most matrices max(A, B) = H, so Eq. 5 and Eq. 4 agree on
    # [H, H]; for [H, 4H] the Eq. 4 update is twice the Eq. 5 one (finding 2)
    lr, wd = 0.1, 0.1
    H = 24
    W0, r4 = _one_step((H, H), 7, lr=lr, weight_decay=wd, scale_mode=orc.SCALE_MAX_DIM)
    _, r5 = _one_step((H, H), 7, lr=lr, weight_decay=wd, scale_mode=orc.SCALE_HIDDEN, hidden_dim=H)
    assert np.max(np.abs(r4.W - r5.W)) < 1e-15
    g = json.load(open(GOLDEN))["mlp_vs_attention_update_ratio"]
    shape = (H, 4 * H)
    W0, r4 = _one_step(shape, 8, lr=lr, weight_decay=wd, scale_mode=orc.SCALE_MAX_DIM)
    _, r5 = _one_step(shape, 8, lr=lr, weight_decay=wd, scale_mode=orc.SCALE_HIDDEN, hidden_dim=H)
    u4, u5 = _update_part(W0, r4, lr, wd), _update_part(W0, r5, lr, wd)
    assert abs(np.linalg.norm(u4) / np.linalg.norm(u5) - g["value"]) < 1e-12


@pytest.mark.parametrize("shape", [(6, 17), (17, 6), (9, 9)])
def test_update_norm_makes_update_rms_exactly_rms_scale(shape):
    lr, wd = 0.05, 0.1
    W0, r = _one_step(shape, 11, lr=lr, weight_decay=wd, scale_mode=orc.SCALE_UPDATE_NORM)
    u = _update_part(W0, r, lr, wd)
    assert abs(math.sqrt(np.mean(u * u)) - 0.2) < 1e-12
    # the logged RMS stays that of O itself
    assert abs(r.rms - math.sqrt(np.mean(r.O * r.O))) < 1e-15


@pytest.mark.parametrize("shape", [(16, 64), (64, 16)])
def test_update_norm_equals_eq4_for_exact_polar_factor(shape):
    # Lemma 1: a full-rank polar factor has RMS 1/sqrt(max(A, B)), so Eq. 6
    # and Eq. 4 give the same step; the cubic iteration (1.5, -0.5, 0) run
    # long reaches the polar factor
    hp = dict(lr=0.1, weight_decay=0.1, ns_steps=60, coeffs=(1.5, -0.5, 0.0))
    _, r4 = _one_step(shape, 21, scale_mode=orc.SCALE_MAX_DIM, **hp)
    _, r6 = _one_step(shape, 21, scale_mode=orc.SCALE_UPDATE_NORM, **hp)
    assert np.max(np.abs(r4.W - r6.W)) < 1e-10


def test_update_norm_zero_gradient_is_pure_decay():
    W0 = rand((5, 7), 31)
    r = orc.muon_step(W0, np.zeros((5, 7)), np.zeros((5, 7)), lr=0.01, weight_decay=0.1,
                      scale_mode=orc.SCALE_UPDATE_NORM)
    assert np.max(np.abs(r.W - (1 - 0.01 * 0.1) * W0)) < 1e-16


# ------------------------------------------------------------------ planted mistakes

def _pins_hold() -> bool:
    """Run a compact subset of the pins; False if any fails or raises."""
    try:
        for shape in [(5, 12), (12, 5), (8, 8)]:
            Y = rand(shape, 1 + shape[0] * 1000 + shape[1])
            if rel_f(orc.newton_schulz(Y, 5), svd_closed_form(Y, 5)) > 1e-12:
                return False
        test_lemma1_full_rank_polar_update_rms((16, 64))
        test_lemma1_full_rank_polar_update_rms((64, 16))
        test_momentum_unrolled_closed_form_and_nesterov_input()
        test_full_step_against_svd_route((12, 20))
        test_full_step_against_svd_route((20, 12))
        test_zero_gradient_is_pure_decoupled_weight_decay()
        test_hidden_dim_scale_matches_eq4_on_square_and_printed_ratio()
        test_update_norm_makes_update_rms_exactly_rms_scale((6, 17))
        test_update_norm_equals_eq4_for_exact_polar_factor((16, 64))
        test_update_norm_zero_gradient_is_pure_decay()
    except Exception:
        return False
    return True


MUTATIONS = {
    "gram_transposed_operand": ("gram", lambda X: np.asarray(X, float).T @ np.asarray(X, float)),
    "poly_sign_of_c": ("poly", lambda A, b, c: b * A - c * (A @ A)),
    "poly_drops_square": ("poly", lambda A, b, c: b * A + c * A),
    "iterate_drops_aX": ("ns_iterate", lambda X, B, a: B @ X),
    "iterate_wrong_side": ("ns_iterate", lambda X, B, a: a * X + X @ B if X.shape[0] == X.shape[1] else (a * X).T),
    "norm_is_max_abs": ("frobenius_normalise",
                        lambda Y: (np.asarray(Y, float) / np.abs(Y).max(), float(np.abs(Y).max()))),
    "no_nesterov": ("nesterov_input", lambda M, G, mu: np.asarray(M, float)),
    "damped_momentum": ("momentum", lambda M, G, mu: mu * np.asarray(M, float) + (1 - mu) * np.asarray(G, float)),
    "scale_uses_min": ("update_scale", lambda r, c, s=0.2: s * math.sqrt(min(r, c))),
    "hidden_scale_without_sqrt": ("update_scale_hidden", lambda H, s=0.2: s * float(H)),
    "update_norm_by_mean_abs": ("update_norm_scale",
                                lambda O, s=0.2: s / float(np.mean(np.abs(O))) if np.any(O) else 0.0),
    "update_norm_inverted": ("update_norm_scale", lambda O, s=0.2: s * orc.update_rms(O)),
    "decay_after_update": ("apply_update",
                           lambda W, O, lr, weight_decay, scale: (np.asarray(W, float) - lr * scale * O) * (1 - lr * weight_decay)),
}


def test_pins_hold_on_the_real_oracle():
    assert _pins_hold()


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(orc, attr, fn)
    assert not _pins_hold(), f"planted mistake {name} went unnoticed"
