"""Seeded synthetic inputs shaped like the models of "Muon is Scalable for LLM
Training" (Moonlight technical report).

This module holds the workload shapes and the random-number recipes only; it
contains none of the optimizer's arithmetic.  The CUDA path (through the
binding), the CPU oracle (through the tests) and the benchmark all draw their
inputs from here, so both sides of every parity check see identical values.

Every tensor is drawn from its own numpy PCG64 stream keyed by
(workload id, tensor kind, matrix index, step), so any single matrix of any
step can be regenerated on its own (the oracle checks samples of the largest
workloads that way).

Distributions (the second argument of N(., .) is a variance):
  W ~ N(0, 0.02^2) fp32, G ~ N(0, 1e-6) rounded to bf16 (std 1e-3).
  Newton-Schulz sweep inputs: P diag(sigma) Q^T + E with P, Q iid N(0, 1) of
  rank 64, sigma_k = (1e-3)^(k/63), E ~ N(0, 1e-4) (std 1e-2), rounded to bf16.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

# tensor kinds (part of every seed key)
KIND_W, KIND_G, KIND_NS_INPUT, KIND_ROUTING, KIND_GAIN = 1, 2, 3, 4, 5

W_STD = 0.02
G_STD = 1e-3
LOWRANK_RANK = 64
LOWRANK_SIGMA_MIN = 1e-3
LOWRANK_NOISE_STD = 1e-2


@dataclass
class Workload:
    """A named list of matrix parameters [rows, cols] plus per-matrix flags."""
    wid: int
    name: str
    shapes: list                      # [(name, rows, cols)]
    zero_grad: set = field(default_factory=set)   # matrix indices whose G is all zero
    steps: int = 1
    excluded_gains: int = 0           # 1-D RMSNorm gains that never enter the step
    gain_size: int = 0

    @property
    def n(self) -> int:
        return len(self.shapes)

    @property
    def elements(self) -> int:
        return sum(r * c for _, r, c in self.shapes)


def _expert_shapes(prefix: str, hidden: int = 2048, inter: int = 1408, routed: int = 64, shared: int = 2):
    out = []
    for e in range(routed + shared):
        tag = f"{prefix}shared{e - routed}" if e >= routed else f"{prefix}expert{e}"
        out.append((f"{tag}.gate", hidden, inter))
        out.append((f"{tag}.up", hidden, inter))
        out.append((f"{tag}.down", inter, hidden))
    return out


def rng_for(wid: int, kind: int, index: int = 0, step: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([wid, kind, index, step])))


def tiny() -> Workload:
    """One fp32 W of shape [256, 128], three consecutive steps."""
    return Workload(1, "tiny_256x128", [("w", 256, 128)], steps=3)


NS_SWEEP_SHAPES = [(1024, 1024), (2048, 2048), (4096, 4096), (8192, 8192), (2048, 8192), (8192, 2048)]


def ns_sweep() -> Workload:
    """Single-matrix Newton-Schulz sweep, square and 1:4 shapes."""
    return Workload(2, "ns_sweep", [(f"ns{r}x{c}", r, c) for r, c in NS_SWEEP_SHAPES], steps=1)


def llama16() -> Workload:
    """Dense Llama-style stack: 16 layers at hidden 2048 with GQA k/v and a
    [H, 4H] MLP: 96 matrices, 10 steps."""
    shapes = []
    for layer in range(16):
        p = f"layer{layer}."
        shapes += [(p + "q", 2048, 2048), (p + "k", 2048, 512), (p + "v", 2048, 512),
                   (p + "o", 2048, 2048), (p + "up", 2048, 8192), (p + "down", 8192, 2048)]
    return Workload(3, "llama16_h2048", shapes, steps=10)


def moe_experts() -> Workload:
    """64 routed + 2 shared experts at hidden 2048, intermediate 1408: 198
    matrices in one grouped step; 10% of the routed experts (6, chosen by seed)
    were not routed and have all-zero gradients."""
    shapes = _expert_shapes("")
    zero_experts = rng_for(4, KIND_ROUTING).choice(64, size=6, replace=False)
    zero = {3 * int(e) + j for e in zero_experts for j in range(3)}
    return Workload(4, "moe_66experts_h2048_i1408", shapes, zero_grad=zero, steps=1)


def mixed8() -> Workload:
    """~16B-total MoE with 8 layers; per layer the attention projections
    [2048,3072], [3072,2048], low-rank KV [2048,512], [512,4096], router
    [2048,64] and 66 experts as above: 1624 matrices, 20 steps.  The 16
    RMSNorm gains (2048 each) are excluded from the step."""
    shapes = []
    for layer in range(8):
        p = f"layer{layer}."
        shapes += [(p + "attn_in", 2048, 3072), (p + "attn_out", 3072, 2048), (p + "kv_down", 2048, 512),
                   (p + "kv_up", 512, 4096), (p + "router", 2048, 64)]
        shapes += _expert_shapes(p)
    return Workload(5, "mixed8_moe16b", shapes, steps=20, excluded_gains=16, gain_size=2048)


WORKLOADS = {"tiny": tiny, "ns_sweep": ns_sweep, "llama16": llama16, "moe": moe_experts, "mixed8": mixed8}


def get(name: str) -> Workload:
    return WORKLOADS[name]()


# ---------------------------------------------------------------- generators

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest-even) and return the raw uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def weight(wl: Workload, index: int) -> np.ndarray:
    """W_0 ~ N(0, 0.02^2), fp32, [rows, cols]."""
    _, r, c = wl.shapes[index]
    return rng_for(wl.wid, KIND_W, index).standard_normal((r, c), dtype=np.float32) * np.float32(W_STD)


def grad_f32(wl: Workload, index: int, step: int) -> np.ndarray:
    """G_t ~ N(0, 1e-6) as fp32 (zero for unrouted experts)."""
    _, r, c = wl.shapes[index]
    if index in wl.zero_grad:
        return np.zeros((r, c), dtype=np.float32)
    return rng_for(wl.wid, KIND_G, index, step).standard_normal((r, c), dtype=np.float32) * np.float32(G_STD)


def grad_bf16(wl: Workload, index: int, step: int) -> np.ndarray:
    """G_t rounded to bf16, returned as uint16 bits."""
    return to_bf16_bits(grad_f32(wl, index, step))


def lowrank_ns_input(wl: Workload, index: int) -> np.ndarray:
    """Newton-Schulz sweep input as bf16 bits: rank-64 signal with singular
    scales decaying geometrically from 1 to 1e-3, plus N(0, 1e-4) noise."""
    _, r, c = wl.shapes[index]
    rng = rng_for(wl.wid, KIND_NS_INPUT, index)
    P = rng.standard_normal((r, LOWRANK_RANK), dtype=np.float32)
    Q = rng.standard_normal((c, LOWRANK_RANK), dtype=np.float32)
    k = np.arange(LOWRANK_RANK, dtype=np.float64)
    sigma = (LOWRANK_SIGMA_MIN ** (k / (LOWRANK_RANK - 1))).astype(np.float32)
    E = rng.standard_normal((r, c), dtype=np.float32) * np.float32(LOWRANK_NOISE_STD)
    Y = (P * sigma[None, :]) @ Q.T + E
    return to_bf16_bits(Y)


def gains(wl: Workload) -> np.ndarray:
    """The excluded 1-D RMSNorm gains, N(1, 0.01^2), [count, size] fp32."""
    rng = rng_for(wl.wid, KIND_GAIN)
    return (1.0 + 0.01 * rng.standard_normal((wl.excluded_gains, wl.gain_size))).astype(np.float32)


def parallel_map(fn, items, threads: int | None = None):
    """Run `fn` over `items` on a thread pool (numpy releases the GIL while
    filling large arrays), preserving order."""
    threads = threads or min(16, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        return list(ex.map(fn, items))
