"""SVD-entropy diagnostic (Sec. 3.4): the CUDA path through the C ABI against
the fp64 oracle.

Bounds, from the arithmetic:
- The Gram matrix is fp64; products of fp32 entries are exact, and the sums
  of n <= 2048 terms are good to about 1e-13 of the largest eigenvalue.
- The Householder reduction to tridiagonal form (fp64) is backward stable:
  T has the eigenvalues of a matrix within a small multiple of m eps ||G||
  of G, about 1e-12 of the largest eigenvalue for m = 1408; bisection on
  the Sturm counts stops at a width of 2 eps ||T||.
- The outputs are fp32: H (|H| <= 1) is rounded to 6e-8 and each singular
  value to 6e-8 relative, so sigma^2 to 1.2e-7 relative.
So H is checked to 2e-7 absolute and sigma^2 to 3e-7 sigma_max^2 per value.
That sigma^2 bound is relative to the largest eigenvalue only: every
eigenvalue carries an absolute error of about 1e-12 sigma_max^2 from the
reduction, so a sigma^2 six decades below the largest is good to about 1e-6
of itself, not to the fp32 rounding.  H, which weighs those values by their
tiny energy share, is unaffected at its 2e-7 bound.
"""

import math

import numpy as np
import pytest
import torch

import oracle.entropy_oracle as ent
from matrix_orthogonalizing_optimizer_muon_b200 import _lib as L
from matrix_orthogonalizing_optimizer_muon_b200 import workloads as wlm
from matrix_orthogonalizing_optimizer_muon_b200.api import EntropyPlan

pytestmark = pytest.mark.gpu

TOL_H = 2e-7
TOL_SIG2 = 3e-7


def _spread(shape, seed, decades):
    # U diag(s) V^T with singular values spread over `decades` decades
    rng = np.random.default_rng(seed)
    m = min(shape)
    U, _ = np.linalg.qr(rng.standard_normal((shape[0], m)))
    V, _ = np.linalg.qr(rng.standard_normal((shape[1], m)))
    s = np.logspace(0, -decades, m)
    return (U * s) @ V.T


def _cases():
    rng = np.random.default_rng(2024)
    out = [
        ("gauss_20x30", rng.standard_normal((20, 30))),
        ("gauss_64x64", rng.standard_normal((64, 64))),
        ("gauss_70x40_tall", rng.standard_normal((70, 40))),
        ("gauss_33x70_ragged", rng.standard_normal((33, 70))),
        ("gauss_130x200", rng.standard_normal((130, 200))),
        ("gauss_300x520", rng.standard_normal((300, 520))),
        ("router_2048x64", 0.02 * rng.standard_normal((2048, 64))),
        ("spread_4_decades_256x384", _spread((256, 384), 5, 4)),
        ("spread_2_decades_300x200", _spread((300, 200), 6, 2)),
        ("rank10_200x300", rng.standard_normal((200, 10)) @ rng.standard_normal((10, 300))),
        ("row_1x50", rng.standard_normal((1, 50))),
        ("col_50x1", rng.standard_normal((50, 1))),
        ("zero_40x50", np.zeros((40, 50))),
        ("equal_sv_96x160", 0.3 * np.linalg.qr(rng.standard_normal((160, 96)))[0].T),
    ]
    return [(name, np.ascontiguousarray(W, dtype=np.float32)) for name, W in out]


def _run(mats, sigma=True):
    plan = EntropyPlan([W.shape for W in mats])
    ws = [torch.from_numpy(W).cuda() for W in mats]
    sig = torch.full((plan.num_singular_values,), float("nan"), device="cuda") if sigma else None
    H = plan.compute(ws, sigma=sig)
    torch.cuda.synchronize()
    st, sweeps = plan.status()
    return plan, ws, H.cpu().numpy().astype(np.float64), (sig.cpu().numpy().astype(np.float64) if sigma else None), st, sweeps


def test_entropy_and_spectrum_match_the_oracle():
    cases = _cases()
    mats = [W for _, W in cases]
    plan, _, H, sig, st, sweeps = _run(mats)
    assert st == L.MUON_OK, (st, sweeps)
    off = 0
    errs = {}
    for (name, W), h, sw in zip(cases, H, sweeps):
        m = min(W.shape)
        want_s = ent.singular_values(W)        # the oracle sees the same fp32 values, in fp64
        want_h = ent.svd_entropy(W)
        got_s = sig[off:off + m]
        off += m
        if math.isnan(want_h):
            assert math.isnan(h), name
        else:
            assert abs(h - want_h) <= TOL_H, (name, h, want_h)
            errs[name] = abs(h - want_h)
        scale = max(want_s[0] ** 2, 1e-300)
        assert np.all(np.diff(got_s) <= 0), name                      # descending
        assert np.max(np.abs(got_s ** 2 - want_s ** 2)) <= TOL_SIG2 * scale, name
        assert 1 <= sw <= 24, (name, sw)
    assert off == plan.num_singular_values


def test_expert_weights_at_full_size():
    # W_0 ~ N(0, 0.02^2) of the 64+2-expert batch: both orientations of the
    # [2048, 1408] expert matrices and a router-sized matrix, in one plan
    wl = wlm.moe_experts()
    idx = [0, 2, 100, 197]
    mats = [wlm.weight(wl, i) for i in idx]
    _, _, H, sig, st, sweeps = _run(mats)
    assert st == L.MUON_OK, sweeps
    off = 0
    for W, h in zip(mats, H):
        m = min(W.shape)
        want_s = ent.singular_values(W)
        assert abs(h - ent.entropy_of_spectrum(want_s)) <= TOL_H
        got = sig[off:off + m]
        off += m
        assert np.max(np.abs(got ** 2 - want_s ** 2)) <= TOL_SIG2 * want_s[0] ** 2


def test_bitwise_reproducible_and_entropy_only_call():
    mats = [W for _, W in _cases()[:8]]
    plan = EntropyPlan([W.shape for W in mats])
    ws = [torch.from_numpy(W).cuda() for W in mats]
    sig1 = torch.empty(plan.num_singular_values, device="cuda")
    sig2 = torch.empty_like(sig1)
    H1 = plan.compute(ws, sigma=sig1).clone()
    H2 = plan.compute(ws, sigma=sig2).clone()
    H3 = plan.compute(ws)  # no spectrum requested
    torch.cuda.synchronize()
    assert torch.equal(H1, H2) and torch.equal(H1, H3)
    assert torch.equal(sig1, sig2)


def test_non_finite_matrix_gives_nan_and_status():
    rng = np.random.default_rng(9)
    good = rng.standard_normal((40, 60)).astype(np.float32)
    bad = rng.standard_normal((50, 30)).astype(np.float32)
    bad[3, 4] = np.nan
    _, _, H, _, st, sweeps = _run([good, bad])
    assert st == L.MUON_ERR_NONFINITE
    assert math.isnan(H[1]) and sweeps[1] == 0
    assert abs(H[0] - ent.svd_entropy(good)) <= TOL_H


def test_argument_errors():
    W = torch.randn(16, 24, device="cuda")
    plan = EntropyPlan([(16, 24)])
    with pytest.raises(ValueError):
        plan.compute([W, W])
    with pytest.raises(ValueError):
        plan.compute([torch.randn(24, 16, device="cuda")])
    # the output may not overlap the input
    flat = torch.zeros(16 * 24 + 8, device="cuda")
    Wv = flat[:16 * 24].view(16, 24)
    with pytest.raises(L.MuonError) as e:
        plan.compute([Wv], H=flat[4:5])
    assert e.value.status == L.MUON_ERR_ALIAS
    with pytest.raises(L.MuonError) as e:
        EntropyPlan([(9000, 9000)])
    assert e.value.status == L.MUON_ERR_UNSUPPORTED


def test_profile_phases():
    mats = [W for _, W in _cases()[:6]]
    plan = EntropyPlan([W.shape for W in mats])
    ws = [torch.from_numpy(W).cuda() for W in mats]
    plan.profile(True)
    plan.compute(ws)
    ms = plan.profile_read()
    assert set(ms) == {"gram", "tridiagonal", "bisection", "entropy"} and all(v > 0 for v in ms.values())
