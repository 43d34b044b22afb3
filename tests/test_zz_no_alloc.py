"""The allocation-free entry point, muon_orthogonalize_noalloc.

It exists for callers that cannot call cudaMalloc (device memory owned by a
framework allocator or a fixed budget, loops that must not allocate after
start-up): all of its scratch is one static device array inside libmuon.
This file is collected last on purpose, so a failure here cannot hide any
other test; it passes both alone in a fresh process and after the rest.

Checked through the C ABI: two calls in a row, each compared with the fp64
CPU oracle's Newton-Schulz on the same bf16 input and with the plan-based
muon_orthogonalize, within the bf16-path tolerance; shapes at the edges of
the fixed scratch (the largest square, the thinnest wide and tall shapes,
ragged row pitches next to the element limit); the size limits, argument
errors and the refusal of a capturing stream.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle.muon_oracle as orc
from matrix_orthogonalizing_optimizer_muon_b200 import _lib as L
from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan

pytestmark = pytest.mark.gpu

ABC = tuple(float(np.float32(v)) for v in (3.4445, -4.7750, 2.0315))
TOL = 3e-2  # relative Frobenius error allowed on the bf16-operand path


def rel_f(a, b) -> float:
    a64 = a.double().cpu().numpy() if isinstance(a, torch.Tensor) else np.asarray(a, np.float64)
    b64 = b.double().cpu().numpy() if isinstance(b, torch.Tensor) else np.asarray(b, np.float64)
    return float(np.linalg.norm(a64 - b64) / np.linalg.norm(b64))


def noalloc(x: torch.Tensor, o: torch.Tensor, steps: int = 5) -> None:
    dt = L.MUON_DT_BF16 if x.dtype == torch.bfloat16 else L.MUON_DT_FP32
    L.muon_orthogonalize_noalloc(x.data_ptr(), o.data_ptr(), x.shape[0], x.shape[1], dt, steps, ABC,
                                 torch.cuda.current_stream().cuda_stream)


def plan_path(x: torch.Tensor, steps: int = 5) -> torch.Tensor:
    out = torch.empty(x.shape, device="cuda")
    plan = MuonPlan([tuple(x.shape)])
    plan.orthogonalize([x], [out], ns_steps=steps, coeffs=ABC)
    torch.cuda.synchronize()
    plan.close()
    return out


def oracle_ns(x: torch.Tensor, steps: int = 5) -> np.ndarray:
    # the exact values the GPU read (bf16 or fp32), widened to fp64
    return orc.newton_schulz(x.double().cpu().numpy(), steps, ABC)


def test_two_calls_in_a_row_match_the_oracle_and_the_plan_entry_point():
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    # first call on a tall matrix, second on a wide one with ragged tiles
    x1 = torch.randn(768, 300, device="cuda", generator=g).to(torch.bfloat16)
    x2 = torch.randn(200, 1000, device="cuda", generator=g).to(torch.bfloat16)
    o1 = torch.full(x1.shape, float("nan"), device="cuda")
    o2 = torch.full(x2.shape, float("nan"), device="cuda")
    noalloc(x1, o1)
    noalloc(x2, o2)
    torch.cuda.synchronize()
    assert torch.isfinite(o1).all() and torch.isfinite(o2).all()
    for x, o in ((x1, o1), (x2, o2)):
        assert rel_f(o, oracle_ns(x)) <= TOL
        assert rel_f(o, plan_path(x)) <= TOL


# in-limit edge shapes: the largest square, the thinnest wide and tall shapes
# at the 8192 side limit, and ragged row pitches just under 2^20 elements
EDGE = [(1024, 1024), (128, 8192), (8192, 128), (1023, 1025), (127, 8191), (8191, 127)]


@pytest.mark.parametrize("shape", EDGE)
def test_edge_shapes_match_the_oracle(shape):
    g = torch.Generator(device="cuda")
    g.manual_seed(shape[0] * 7 + shape[1])
    x = torch.randn(shape, device="cuda", generator=g).to(torch.bfloat16)
    o = torch.full(shape, float("nan"), device="cuda")
    noalloc(x, o)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all()
    assert rel_f(o, oracle_ns(x)) <= TOL


def test_repeated_call_is_reproducible_and_fp32_input_accepted():
    g = torch.Generator(device="cuda")
    g.manual_seed(6)
    x = torch.randn(512, 512, device="cuda", generator=g)
    a = torch.empty_like(x)
    b = torch.empty_like(x)
    noalloc(x, a)
    noalloc(x, b)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert rel_f(a, oracle_ns(x)) <= TOL
    assert rel_f(a, plan_path(x)) <= TOL


def test_limits_and_argument_errors():
    lib = L.load()
    abc = (ctypes.c_float * 3)(*ABC)
    x = torch.zeros(4, 4, device="cuda", dtype=torch.bfloat16)
    o = torch.zeros(4, 4, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    xp, op = ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(o.data_ptr())
    # beyond the static scratch: more than 2^20 elements, a side above 8192, min side above 1024
    assert lib.muon_orthogonalize_noalloc(xp, op, 2048, 1024, 0, 5, abc, s) == L.MUON_ERR_UNSUPPORTED
    assert lib.muon_orthogonalize_noalloc(xp, op, 16, 8193, 0, 5, abc, s) == L.MUON_ERR_UNSUPPORTED
    assert lib.muon_orthogonalize_noalloc(xp, op, 1025, 1025, 0, 5, abc, s) == L.MUON_ERR_UNSUPPORTED
    assert lib.muon_orthogonalize_noalloc(None, op, 4, 4, 0, 5, abc, s) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_orthogonalize_noalloc(xp, op, 0, 4, 0, 5, abc, s) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_orthogonalize_noalloc(xp, op, 4, 4, 7, 5, abc, s) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_orthogonalize_noalloc(xp, xp, 4, 4, 0, 5, abc, s) == L.MUON_ERR_ALIAS


def test_capturing_stream_is_refused_and_nothing_is_enqueued():
    lib = L.load()
    abc = (ctypes.c_float * 3)(*ABC)
    x = torch.randn(64, 96, device="cuda").to(torch.bfloat16)
    o = torch.zeros(64, 96, device="cuda")
    noalloc(x, o)  # the device is set up before any capture
    torch.cuda.synchronize()
    before = o.clone()
    graph = torch.cuda.CUDAGraph()
    codes = []
    with torch.cuda.graph(graph):
        s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        codes.append(lib.muon_orthogonalize_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                                    64, 96, L.MUON_DT_BF16, 5, abc, s))
        x.mul_(1.0)  # the capture holds one ordinary node
    graph.replay()
    torch.cuda.synchronize()
    assert codes == [L.MUON_ERR_UNSUPPORTED]
    assert torch.equal(o, before)
    del graph
    # the entry point still works after the refused call
    o2 = torch.empty_like(o)
    noalloc(x, o2)
    torch.cuda.synchronize()
    assert torch.equal(o2, before)


def test_zero_input_after_nonzero_gives_exact_zero_output():
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    x = torch.randn(300, 520, device="cuda", generator=g).to(torch.bfloat16)
    o = torch.empty(x.shape, device="cuda")
    noalloc(x, o)
    torch.cuda.synchronize()
    assert bool(o.abs().max() > 0)
    x.zero_()
    noalloc(x, o)
    torch.cuda.synchronize()
    assert torch.equal(o, torch.zeros_like(o))
