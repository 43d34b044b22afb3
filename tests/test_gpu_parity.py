"""GPU (CUDA path through the C ABI) against the fp64 CPU oracle.

Every comparison uses identical seeded inputs on both sides and the
thresholds of the acceptance criteria: relative Frobenius error of O at most
3e-2 on the bf16-operand path and 1e-4 on the fp32 path, momentum within
1e-6 relative, and max |dW_gpu - dW_oracle| <= 2e-2 lr 0.2 sqrt(max(A, B))
with the oracle started from the GPU's own W_{t-1} and M_{t-1}.
"""

import numpy as np
import pytest
import torch

import oracle.muon_oracle as orc
from matrix_orthogonalizing_optimizer_muon_b200 import workloads as wlm
from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan

from _gpu import (ABC32, LR, MU, TOL_O_BF16, TOL_O_FP32, WD, assert_step_errors, bf16_cuda, check_step, f32, host32,
                  host64, random_bf16, rel_f)
from _oracle_pool import OraclePool

pytestmark = pytest.mark.gpu

# odd and tile-straddling shapes: several 128x256 tiles plus ragged tails,
# wide and tall, K not a multiple of 64, rank-1 rows/columns
SMALL = [(128, 128), (256, 128), (128, 256), (200, 136), (136, 200), (1, 7), (7, 1), (64, 640), (640, 64),
         (300, 520), (520, 300), (384, 384), (17, 1000), (1000, 17)]

CASES = {
    "gram_update": (1, (0.0, 1.0, 0.0)),    # X1 = (X X^T) X: Gram + X-update kernels
    "poly_only": (1, (0.0, 0.0, 1.0)),      # X1 = (X X^T)^2 X: adds the A A product
    "quintic_5": (5, ABC32),                # the method's iteration
    "no_iteration": (0, ABC32),             # O = Y / ||Y||_F
    "cubic_3": (3, (1.5, -0.5, 0.0)),       # b A term only, several iterations
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_orthogonalize_small_shapes_grouped(case, precision):
    steps, abc = CASES[case]
    abc = tuple(f32(v) for v in abc)
    xs, hosts = [], []
    for k, shp in enumerate(SMALL):
        x, h = random_bf16(shp, 1000 + k)
        xs.append(x)
        hosts.append(h)
    outs = [torch.full(s, float("nan"), device="cuda") for s in SMALL]
    plan = MuonPlan(SMALL, fp32_ns=(precision == "fp32"))
    plan.orthogonalize(xs, outs, ns_steps=steps, coeffs=abc, precision=precision)
    torch.cuda.synchronize()
    assert plan.status() == 0
    tol = TOL_O_FP32 if precision == "fp32" else TOL_O_BF16
    errs = {}
    for shp, h, o in zip(SMALL, hosts, outs):
        want = orc.newton_schulz(h, steps, abc)
        errs[shp] = rel_f(host64(o), want)
    worst = max(errs.values())
    assert worst <= tol, errs


@pytest.mark.parametrize("shape", [(1024, 1024), (2048, 512), (512, 2048), (1408, 2048), (2048, 1408)])
def test_orthogonalize_medium_lowrank(shape):
    # the sweep's low-rank-plus-noise structure at sizes the oracle finishes fast
    wl = wlm.Workload(90, "medium", [("x", *shape)])
    bits = wlm.lowrank_ns_input(wl, 0)
    x = bf16_cuda(bits)
    h = wlm.bf16_bits_to_f32(bits).astype(np.float64)
    out = torch.empty(shape, device="cuda")
    plan = MuonPlan([shape])
    plan.orthogonalize([x], [out], ns_steps=5, coeffs=ABC32)
    want = orc.newton_schulz(h, 5, ABC32)
    err = rel_f(host64(out), want)
    assert err <= TOL_O_BF16, err


@pytest.mark.parametrize("g_dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_tiny_three_steps(g_dtype, precision):
    """The tiny workload: one [256, 128] fp32 W, 3 consecutive steps."""
    wl = wlm.tiny()
    W = torch.from_numpy(wlm.weight(wl, 0)).cuda()
    M = torch.empty_like(W)
    plan = MuonPlan([W.shape], momenta=[M], fp32_ns=(precision == "fp32"))
    rms = torch.zeros(1, device="cuda")
    # the fp32 path is checked with a larger learning rate so that rounding of
    # W itself (fp32) stays far below the 1e-4 criterion on O
    lr = LR if precision == "bf16" else f32(0.05)
    for t in range(wl.steps):
        if g_dtype == "bf16":
            bits = wlm.grad_bf16(wl, 0, t)
            G = bf16_cuda(bits)
            G64 = wlm.bf16_bits_to_f32(bits).astype(np.float64)
        else:
            g = wlm.grad_f32(wl, 0, t)
            G = torch.from_numpy(g).cuda()
            G64 = g.astype(np.float64)
        W_prev, M_prev = host64(W), host64(M)
        plan.step([(W, G, M)], lr=lr, weight_decay=WD, momentum=MU, coeffs=ABC32, precision=precision,
                  update_rms=rms)
        torch.cuda.synchronize()
        check_step(W_prev, M_prev, G64, host64(W), host64(M), float(rms.item()), lr=lr, wd=WD, mu=MU,
                   precision=precision)
    assert plan.status() == 0


def test_plain_momentum_and_zero_iterations():
    wl = wlm.tiny()
    W = torch.from_numpy(wlm.weight(wl, 0)).cuda()
    M = torch.zeros_like(W)
    G = bf16_cuda(wlm.grad_bf16(wl, 0, 0))
    plan = MuonPlan([W.shape])
    for nest, steps in [(False, 5), (True, 0), (False, 0)]:
        W_prev, M_prev = host64(W), host64(M)
        plan.step([(W, G, M)], lr=LR, weight_decay=WD, momentum=MU, ns_steps=steps, coeffs=ABC32, nesterov=nest)
        torch.cuda.synchronize()
        check_step(W_prev, M_prev, host64(G), host64(W), host64(M), None, lr=LR, wd=WD, mu=MU, ns_steps=steps,
                   nesterov=nest)


def test_zero_gradient_matrix_is_pure_decay():
    shapes = [(256, 128), (128, 256), (300, 200)]
    Ws = [torch.randn(s, device="cuda") * 0.02 for s in shapes]
    Ms = [torch.zeros(s, device="cuda") for s in shapes]
    Gs = [torch.zeros(s, device="cuda", dtype=torch.bfloat16) for s in shapes]
    Gs[1].normal_(0, 1e-3)
    plan = MuonPlan(shapes)
    rms = torch.full((3,), -1.0, device="cuda")
    W0 = [host64(w) for w in Ws]
    plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32, update_rms=rms)
    torch.cuda.synchronize()
    for k in (0, 2):
        want = W0[k] - LR * (WD * W0[k])
        # two fp32 roundings of the decay product and one of the result
        assert np.max(np.abs(host64(Ws[k]) - want) / np.maximum(np.abs(want), 1e-30)) <= 3 * 2.0 ** -24
        assert float(rms[k]) == 0.0
    assert float(rms[1]) > 0


def test_moe_expert_batch_full_size_every_matrix():
    """The 64+2-expert batch (198 matrices, one grouped call, the launch
    configuration the benchmark times): W, M, O and the update RMS of every
    matrix, the 18 unrouted ones included, against the oracle."""
    wl = wlm.moe_experts()
    shapes = [(r, c) for _, r, c in wl.shapes]
    Ws = [torch.from_numpy(wlm.weight(wl, i)).cuda() for i in range(wl.n)]
    Gs = [bf16_cuda(wlm.grad_bf16(wl, i, 0)) for i in range(wl.n)]
    Ms = [torch.empty(s, device="cuda") for s in shapes]
    plan = MuonPlan(shapes, momenta=Ms)
    rms = torch.zeros(wl.n, device="cuda")
    plan.step(list(zip(Ws, Gs, Ms)), lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32, update_rms=rms)
    torch.cuda.synchronize()
    assert plan.status() == 0
    rms_h = rms.cpu().numpy()
    with OraclePool() as pool:
        for i in range(wl.n):
            pool.submit_step(i, wlm.weight(wl, i), np.zeros(shapes[i], np.float32),
                             wlm.bf16_bits_to_f32(wlm.grad_bf16(wl, i, 0)), host32(Ws[i]), host32(Ms[i]),
                             float(rms_h[i]), lr=LR, wd=WD, mu=MU, coeffs=ABC32)
        res = pool.drain()
    assert sorted(r["key"] for r in res) == list(range(wl.n))
    for r in res:
        assert_step_errors(r)
    nz = [r for r in res if r["key"] not in wl.zero_grad]
    worst = {"O": max(r["O"] for r in nz), "dW/bound": max(r["dW"] / r["dW_bound"] for r in res),
             "M": max(r["M"] for r in res), "rms": max(r["rms"] for r in nz)}
    print("moe worst", worst)
    plan.close()
