"""SVD-entropy diagnostic (Sec. 3.4): relative accuracy of the small singular
values, which the H and sigma_max-relative bounds of test_gpu_entropy.py do
not resolve.

Bounds, from the arithmetic of the fp64 path:
- G = X X^T from fp32 entries: products are exact, each sum of n terms
  rounds to within n eps |x_i| |x_j| <= n eps sigma_max^2 per entry.
- The Householder reduction is backward stable: T has the eigenvalues of a
  symmetric matrix within c m eps ||G|| of G (Golub and Van Loan, Sec. 8.3.1),
  so every eigenvalue moves by at most that much (Weyl); bisection adds
  2 eps ||T||.
- The fp32 output rounds sigma to 6e-8 relative, sigma^2 to 1.2e-7.
With c = 8, an eigenvalue lambda is good to
  rel(lambda) <= 1.2e-7 + 8 (m + n) eps sigma_max^2 / lambda.
For singular values spread over two decades (sigma^2 down to 1e-4 of the
largest, m + n = 500) that is about 1.3e-7 at every value; over four decades
(sigma^2 down to 1e-8, m + n = 640) it is about 1.1e-4 at the smallest value
and 1.3e-7 at the largest.  The oracle (LAPACK SVD of the same
fp32 matrix in fp64) is accurate to eps sigma_max per singular value.
"""

import numpy as np
import pytest
import torch

import oracle.entropy_oracle as ent
from matrix_orthogonalizing_optimizer_muon_b200 import _lib as L
from matrix_orthogonalizing_optimizer_muon_b200.api import EntropyPlan

pytestmark = pytest.mark.gpu

EPS = np.finfo(np.float64).eps


def _spread(shape, seed, decades):
    rng = np.random.default_rng(seed)
    m = min(shape)
    U, _ = np.linalg.qr(rng.standard_normal((shape[0], m)))
    V, _ = np.linalg.qr(rng.standard_normal((shape[1], m)))
    s = np.logspace(0, -decades, m)
    return np.ascontiguousarray((U * s) @ V.T, dtype=np.float32)


@pytest.mark.parametrize("shape,decades,seed", [((200, 300), 2, 31), ((256, 384), 4, 32), ((384, 256), 4, 33),
                                                ((700, 500), 3, 34)])
def test_small_singular_values_to_relative_accuracy(shape, decades, seed):
    W = _spread(shape, seed, decades)
    plan = EntropyPlan([W.shape])
    sig = torch.empty(plan.num_singular_values, device="cuda")
    plan.compute([torch.from_numpy(W).cuda()], sigma=sig)
    torch.cuda.synchronize()
    st, done = plan.status()
    assert st == L.MUON_OK and done == [1]
    got = sig.cpu().numpy().astype(np.float64) ** 2
    want = ent.singular_values(W) ** 2
    m, n = min(shape), max(shape)
    bound = 1.2e-7 + 8 * (m + n) * EPS * want[0] / want
    rel = np.abs(got - want) / want
    assert np.all(rel <= bound), (float(np.max(rel / bound)), int(np.argmax(rel / bound)))
    plan.close()


def test_large_batch_runs_one_cta_per_matrix():
    """160 matrices do not fit as clusters of two CTAs on separate SMs, so the
    reduction runs one CTA per matrix (the path of the MoE-sized batches);
    the plans of the other tests here hold one matrix each (clusters of up
    to 16 CTAs).  Same bounds as test_gpu_entropy.py: H to 2e-7 and sigma^2
    to 3e-7 sigma_max^2."""
    rng = np.random.default_rng(41)
    mats = [np.ascontiguousarray(rng.standard_normal((40 + (i % 7) * 13, 60 + (i % 5) * 17)), dtype=np.float32)
            for i in range(160)]
    plan = EntropyPlan([W.shape for W in mats])
    sig = torch.empty(plan.num_singular_values, device="cuda")
    H = plan.compute([torch.from_numpy(W).cuda() for W in mats], sigma=sig)
    torch.cuda.synchronize()
    st, done = plan.status()
    assert st == L.MUON_OK and done == [1] * len(mats)
    H = H.cpu().numpy().astype(np.float64)
    got = sig.cpu().numpy().astype(np.float64)
    off = 0
    for W, h in zip(mats, H):
        m = min(W.shape)
        want = ent.singular_values(W)
        assert abs(h - ent.entropy_of_spectrum(want)) <= 2e-7
        assert np.max(np.abs(got[off:off + m] ** 2 - want ** 2)) <= 3e-7 * want[0] ** 2
        off += m
    plan.close()


def test_cluster_size_follows_the_plan_and_results_agree():
    """The reduction's cluster size shrinks as the plan grows (up to 16 CTAs
    per matrix for a few matrices, one CTA per matrix for large batches;
    clusters are used only when all of them fit at once with one CTA per
    SM).  One matrix computed inside plans of different sizes matches the
    oracle's H and spectrum every time, whatever the cluster size."""
    rng = np.random.default_rng(51)
    W0 = np.ascontiguousarray(rng.standard_normal((300, 520)), dtype=np.float32)
    want = ent.singular_values(W0)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    sizes = []
    for count in (1, 6, 30, 40, 160):
        mats = [W0] + [np.ascontiguousarray(rng.standard_normal((48, 80)), dtype=np.float32)
                       for _ in range(count - 1)]
        plan = EntropyPlan([W.shape for W in mats])
        c = plan.cluster_size
        assert c in (1, 2, 4, 8, 16)
        assert c == 1 or c * count <= sms, (count, c)
        sizes.append(c)
        sig = torch.empty(plan.num_singular_values, device="cuda")
        H = plan.compute([torch.from_numpy(W).cuda() for W in mats], sigma=sig)
        torch.cuda.synchronize()
        assert plan.status()[0] == L.MUON_OK
        assert abs(float(H[0]) - ent.entropy_of_spectrum(want)) <= 2e-7, (count, c)
        got = sig[:min(W0.shape)].cpu().numpy().astype(np.float64)
        assert np.max(np.abs(got ** 2 - want ** 2)) <= 3e-7 * want[0] ** 2, (count, c)
        plan.close()
    assert sizes == sorted(sizes, reverse=True), sizes
    assert sizes[0] >= 8 and sizes[-1] == 1, sizes
    assert len(set(sizes)) >= 3, sizes  # several cluster sizes were exercised
