"""Pins of the AdamW oracle (no GPU): a library routine, closed forms, and
the update-RMS property the pages state for Adam/AdamW."""

import math

import numpy as np
import pytest
import torch

import oracle.adamw_oracle as ado


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("decay", [True, False])
def test_matches_torch_adamw_in_float64(decay):
    # torch.optim.AdamW (decoupled decay, bias correction) as the library routine
    shape, T = (7, 13), 6
    lr, wd, betas, eps = 3e-3, 0.1, (0.9, 0.95), 1e-8
    P0 = rand(shape, 1)
    Gs = [rand(shape, 10 + t, 1e-2) for t in range(T)]
    p = torch.tensor(P0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([p], lr=lr, betas=betas, eps=eps, weight_decay=wd if decay else 0.0)
    P, m, v = P0, np.zeros(shape), np.zeros(shape)
    for t in range(T):
        p.grad = torch.tensor(Gs[t], dtype=torch.float64)
        opt.step()
        r = ado.adamw_step(P, Gs[t], m, v, step=t + 1, lr=lr, weight_decay=wd, betas=betas, eps=eps, decay=decay)
        P, m, v = r.P, r.m, r.v
        assert np.max(np.abs(P - p.detach().numpy())) < 1e-14
        st = opt.state[p]
        assert np.max(np.abs(m - st["exp_avg"].numpy())) < 1e-16
        assert np.max(np.abs(v - st["exp_avg_sq"].numpy())) < 1e-18


def test_first_step_is_sign_like_with_update_rms_one():
    # t = 1: m_hat = g, v_hat = g^2, so the update is g / (|g| + eps): the
    # update RMS is ~1, the property Sec. 2.2 quotes for Adam and AdamW
    G = rand((64, 64), 3, 1e-3)
    r = ado.adamw_step(np.zeros_like(G), G, np.zeros_like(G), np.zeros_like(G), step=1, lr=1.0, weight_decay=0.0)
    assert np.max(np.abs(r.update - G / (np.abs(G) + 1e-8))) < 1e-15
    assert abs(ado.update_rms(r.update) - 1.0) < 1e-2  # "about 1": tiny |g| near eps pull it down slightly


def test_constant_gradient_closed_form():
    # with g constant the bias-corrected moments are exactly g and g^2 at every t
    g, T = 0.37, 9
    P, m, v = np.array([1.0]), np.zeros(1), np.zeros(1)
    for t in range(1, T + 1):
        r = ado.adamw_step(P, np.array([g]), m, v, step=t, lr=0.01, weight_decay=0.0, eps=0.0)
        assert abs(r.m[0] - g * (1 - 0.9 ** t)) < 1e-15
        assert abs(r.update[0] - 1.0) < 1e-13
        P, m, v = r.P, r.m, r.v
    assert abs(P[0] - (1.0 - 0.01 * T)) < 1e-13


def test_zero_gradient_is_pure_decay_and_opt_out():
    P0 = rand((5,), 4)
    z = np.zeros(5)
    r = ado.adamw_step(P0, z, z, z, step=1, lr=0.1, weight_decay=0.2)
    assert np.max(np.abs(r.P - P0 * (1 - 0.02))) < 1e-16
    r = ado.adamw_step(P0, z, z, z, step=1, lr=0.1, weight_decay=0.2, decay=False)
    assert np.array_equal(r.P, P0)


def test_rejects_step_zero():
    with pytest.raises(ValueError):
        ado.adamw_step(np.zeros(2), np.zeros(2), np.zeros(2), np.zeros(2), step=0, lr=1.0, weight_decay=0.0)


def _torch_reference(P0, Gs, lr, wd, betas, eps):
    p = torch.tensor(P0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([p], lr=lr, betas=betas, eps=eps, weight_decay=wd)
    for G in Gs:
        p.grad = torch.tensor(G, dtype=torch.float64)
        opt.step()
    return p.detach().numpy()


MUTANTS = {
    # each is a plausible mistake in the update; the library pin must reject it
    "no_bias_correction": lambda m, v, t, b1, b2, eps: m / (np.sqrt(v) + eps),
    "eps_inside_sqrt": lambda m, v, t, b1, b2, eps: (m / (1 - b1 ** t)) / np.sqrt(v / (1 - b2 ** t) + eps),
    "betas_swapped": lambda m, v, t, b1, b2, eps: (m / (1 - b2 ** t)) / (np.sqrt(v / (1 - b1 ** t)) + eps),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_library_pin_rejects_planted_mistakes(name, monkeypatch):
    shape, lr, wd, betas, eps = (6, 5), 3e-3, 0.1, (0.9, 0.95), 1e-8
    P0 = rand(shape, 1)
    Gs = [rand(shape, 20 + t, 1e-2) for t in range(4)]
    want = _torch_reference(P0, Gs, lr, wd, betas, eps)
    mut = MUTANTS[name]
    real_sqrt = np.sqrt

    def mutated_step(P, G, m_prev, v_prev, *, step, lr, weight_decay, betas=betas, eps=eps, decay=True):
        b1, b2 = betas
        m = b1 * m_prev + (1 - b1) * G
        v = b2 * v_prev + (1 - b2) * G * G
        u = mut(m, v, step, b1, b2, eps)
        return ado.AdamWResult(P=P - lr * (u + weight_decay * P), m=m, v=v, update=u)

    monkeypatch.setattr(ado, "adamw_step", mutated_step)
    P, m, v = P0, np.zeros(shape), np.zeros(shape)
    for t, G in enumerate(Gs):
        r = ado.adamw_step(P, G, m, v, step=t + 1, lr=lr, weight_decay=wd)
        P, m, v = r.P, r.m, r.v
    assert np.max(np.abs(P - want)) > 1e-9, name
    assert real_sqrt is np.sqrt
