"""Row-by-row checks of the symmetric products (X X^T and A A).

The symmetric outputs are written one 32 x 32 block at a time, each block
together with its mirror.  When the last row block of a matrix is ragged,
its off-diagonal tiles are computed transposed (rows of a full block,
columns of the ragged one).  A block that the kernel failed to write, or
wrote to the wrong place, would move the relative Frobenius error of a
1408 x 1408 product by about 2%.  Checked row by row it moves that row by
about 10%.  So these tests compare every output row after one iteration
with the fp64 oracle:
- the Gram product followed by the X update, X1 = (X X^T) X;
- the Gram product, then the A A product, then the update, X1 = (X X^T)^2 X.
Before the checked call, the same plan runs once on other data, so a block
that is never written holds stale values and fails.

The last row block has 44, 188, 232, 128 and 256 (full) rows for
m = 300, 700, 1000, 1408 and 512, in both orientations.
"""

import numpy as np
import pytest
import torch

import oracle.muon_oracle as orc
from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan

from _gpu import ABC32, TOL_O_BF16, f32, host64, random_bf16, rel_f

pytestmark = pytest.mark.gpu

SHAPES = [(300, 420), (420, 300), (700, 900), (900, 700), (1000, 1100), (1100, 1000), (1408, 2048),
          (2048, 1408), (512, 600)]

# One iteration rounds A (and A A) to bf16 once; a row's relative error is a
# few times 2^-9 with all blocks right.  A missing off-diagonal block of A
# removes a term of about sqrt(32 / m) of the row.
TOL_ROW = 1.5e-2


def _row_errors(got, want):
    d = np.linalg.norm(want, axis=1)
    return np.linalg.norm(got - want, axis=1) / np.maximum(d, 1e-300)


@pytest.mark.parametrize("coeffs", [(0.0, 1.0, 0.0), (0.0, 0.0, 1.0)], ids=["gram_update", "poly"])
def test_symmetric_products_row_by_row(coeffs):
    abc = tuple(f32(v) for v in coeffs)
    plan = MuonPlan(SHAPES)
    # a first call on other data leaves every workspace block holding stale values
    xs0 = [random_bf16(s, 500 + k, scale=3.0)[0] for k, s in enumerate(SHAPES)]
    outs = [torch.empty(s, device="cuda") for s in SHAPES]
    plan.orthogonalize(xs0, outs, ns_steps=1, coeffs=abc)
    xs, hosts = [], []
    for k, s in enumerate(SHAPES):
        x, h = random_bf16(s, 600 + k)
        xs.append(x)
        hosts.append(h)
    outs = [torch.full(s, float("nan"), device="cuda") for s in SHAPES]
    plan.orthogonalize(xs, outs, ns_steps=1, coeffs=abc)
    torch.cuda.synchronize()
    assert plan.status() == 0
    worst = {}
    for s, h, o in zip(SHAPES, hosts, outs):
        got = host64(o)
        want = orc.newton_schulz(h, 1, abc)
        # rows of the wide orientation: the short side indexes the symmetric product
        if s[0] > s[1]:
            got, want = got.T, want.T
        e = _row_errors(got, want)
        worst[s] = float(e.max())
    assert max(worst.values()) <= TOL_ROW, worst


@pytest.mark.parametrize("split", [2, 4])
def test_split_k_gram_row_by_row(split, monkeypatch):
    """One matrix per plan with the Gram product's K range split into parts
    (fp32 partial products and a fixed-order reduction).  Plans choose the
    split for single matrices with a long K (2048 x 8192 takes 2 parts);
    MUON_SPLITK forces it here on every shape.  Same row-by-row check of
    X1 = (X X^T) X, and a repeated call is bitwise equal."""
    monkeypatch.setenv("MUON_SPLITK", str(split))
    abc = tuple(f32(v) for v in (0.0, 1.0, 0.0))
    worst = {}
    for k, s in enumerate(SHAPES):
        plan = MuonPlan([s])
        x, h = random_bf16(s, 800 + k)
        o1 = torch.full(s, float("nan"), device="cuda")
        o2 = torch.full(s, float("nan"), device="cuda")
        plan.orthogonalize([x], [o1], ns_steps=1, coeffs=abc)
        plan.orthogonalize([x], [o2], ns_steps=1, coeffs=abc)
        torch.cuda.synchronize()
        assert plan.status() == 0
        assert torch.equal(o1, o2)
        got, want = host64(o1), orc.newton_schulz(h, 1, abc)
        if s[0] > s[1]:
            got, want = got.T, want.T
        worst[s] = float(_row_errors(got, want).max())
        plan.close()
    assert max(worst.values()) <= TOL_ROW, worst
    # and the method's five iterations on the same plans, within the acceptance bound
    errs = {}
    for k, s in enumerate(SHAPES):
        plan = MuonPlan([s])
        x, h = random_bf16(s, 900 + k)
        o = torch.full(s, float("nan"), device="cuda")
        plan.orthogonalize([x], [o], ns_steps=5, coeffs=ABC32)
        torch.cuda.synchronize()
        errs[s] = rel_f(host64(o), orc.newton_schulz(h, 5, ABC32))
        plan.close()
    assert max(errs.values()) <= TOL_O_BF16, errs


@pytest.mark.parametrize("levels", [1, 2])
@pytest.mark.parametrize("coeffs", [(0.0, 1.0, 0.0), (0.0, 0.0, 1.0)], ids=["gram_update", "poly"])
def test_n_split_tiles_row_by_row(levels, coeffs, monkeypatch):
    """The symmetric and X-update tiles split along N (256 -> 128 -> 64
    columns), which plans with few tiles choose (one 2048 x 2048 matrix
    splits its symmetric tiles once, one 1024 x 1024 matrix every list
    twice); MUON_NSPLIT forces it here on the whole multi-shape plan.  Same
    stale-workspace and row-by-row check as above."""
    monkeypatch.setenv("MUON_NSPLIT", str(levels))
    abc = tuple(f32(v) for v in coeffs)
    plan = MuonPlan(SHAPES)
    xs0 = [random_bf16(s, 1500 + k, scale=3.0)[0] for k, s in enumerate(SHAPES)]
    plan.orthogonalize(xs0, [torch.empty(s, device="cuda") for s in SHAPES], ns_steps=1, coeffs=abc)
    xs, hosts = [], []
    for k, s in enumerate(SHAPES):
        x, h = random_bf16(s, 1600 + k)
        xs.append(x)
        hosts.append(h)
    outs = [torch.full(s, float("nan"), device="cuda") for s in SHAPES]
    plan.orthogonalize(xs, outs, ns_steps=1, coeffs=abc)
    torch.cuda.synchronize()
    assert plan.status() == 0
    worst = {}
    for s, h, o in zip(SHAPES, hosts, outs):
        got, want = host64(o), orc.newton_schulz(h, 1, abc)
        if s[0] > s[1]:
            got, want = got.T, want.T
        worst[s] = float(_row_errors(got, want).max())
    assert max(worst.values()) <= TOL_ROW, worst
    plan.close()


def test_symmetric_tiles_five_iterations():
    """The method's five iterations on the same shapes, within the acceptance bound."""
    plan = MuonPlan(SHAPES)
    xs, hosts = [], []
    for k, s in enumerate(SHAPES):
        x, h = random_bf16(s, 700 + k)
        xs.append(x)
        hosts.append(h)
    outs = [torch.full(s, float("nan"), device="cuda") for s in SHAPES]
    plan.orthogonalize(xs, outs, ns_steps=5, coeffs=ABC32)
    torch.cuda.synchronize()
    assert plan.status() == 0
    errs = {s: rel_f(host64(o), orc.newton_schulz(h, 5, ABC32)) for s, h, o in zip(SHAPES, hosts, outs)}
    assert max(errs.values()) <= TOL_O_BF16, errs

