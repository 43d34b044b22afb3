"""Data-parallel Muon (owner-partitioned form of "Muon is Scalable for LLM
Training", Sec. 2.3, Algorithm 1) on two gloo ranks on CPU.  The owners'
local step is the fp64 oracle here (the product's default is libmuon on the
GPU); what is under test is the partition, the gradient reduction, the
momentum ownership and the weight all-gather."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.muon_oracle as orc
from matrix_orthogonalizing_optimizer_muon_b200.distributed import DistributedMuon, assign_owners, assign_waves, ns_work

SHAPES = [(24, 40), (40, 24), (16, 16), (8, 64), (33, 17)]
LR, WD, MU = 0.05, 0.1, 0.95
STEPS = 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def oracle_local_step(params, *, lr, weight_decay, momentum):
    """Owner step on CPU tensors: the fp64 oracle, results rounded to fp32."""
    rms = []
    for W, G, M in params:
        r = orc.muon_step(W.double().numpy(), G.double().numpy(), M.double().numpy(), lr=lr,
                          weight_decay=weight_decay, momentum_coef=momentum)
        W.copy_(torch.from_numpy(r.W))
        M.copy_(torch.from_numpy(r.M))
        rms.append(r.rms)
    return torch.tensor(rms, dtype=torch.float32)


def grads(rank, step):
    g = torch.Generator().manual_seed(1000 * rank + step)
    return [torch.randn(s, generator=g) * 1e-3 for s in SHAPES]


def weights():
    g = torch.Generator().manual_seed(7)
    return [torch.randn(s, generator=g) * 0.02 for s in SHAPES]


def _worker(rank, world, port, out, waves=2):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        opt = DistributedMuon(SHAPES, local_step=oracle_local_step, device="cpu", waves=waves)
        Ws = weights()
        rms = None
        for t in range(STEPS):
            rms = opt.step(list(zip(Ws, grads(rank, t))), lr=LR, weight_decay=WD, momentum=MU).clone()
        out.put((rank, [W.numpy().copy() for W in Ws], rms.numpy().copy(), sorted(opt.M), opt.owner))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("waves", [1, 2, 3])
def test_two_ranks_match_a_single_process_step_on_the_summed_gradient(waves):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, waves)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # reference: one process, the gradient summed over the two ranks (fp32, one rounding)
    Ws = weights()
    Ms = [torch.zeros(s) for s in SHAPES]
    for t in range(STEPS):
        Gsum = [a + b for a, b in zip(grads(0, t), grads(1, t))]
        ref_rms = oracle_local_step(list(zip(Ws, Gsum, Ms)), lr=LR, weight_decay=WD, momentum=MU)
    for rank, W_out, rms, owned, owner in res:
        for a, b in zip(W_out, Ws):
            assert np.array_equal(a, b.numpy())          # every rank ends with identical weights
        assert np.array_equal(rms, ref_rms.numpy())
        assert owned == [i for i, r in enumerate(owner) if r == rank]   # momentum only on the owner
    owners = res[0][4]
    assert set(owners) == {0, 1}


def test_owner_assignment_is_balanced_and_deterministic():
    shapes = [(2048, 1408)] * 7 + [(1408, 2048)] * 5 + [(512, 512)] * 3
    for world in (1, 2, 3, 8):
        a = assign_owners(shapes, world)
        assert a == assign_owners(list(shapes), world)
        load = [sum(ns_work(s) for s, r in zip(shapes, a) if r == k) for k in range(world)]
        assert max(load) - min(load) <= max(ns_work(s) for s in shapes)


def test_waves_split_each_rank_evenly_and_deterministically():
    shapes = [(2048, 1408)] * 9 + [(1408, 2048)] * 6 + [(512, 512)] * 4 + [(2048, 64)] * 3
    for world in (1, 2, 4):
        owner = assign_owners(shapes, world)
        for waves in (1, 2, 3):
            w = assign_waves(shapes, owner, world, waves)
            assert w == assign_waves(list(shapes), list(owner), world, waves)
            assert all(0 <= k < waves for k in w)
            for r in range(world):
                load = [sum(ns_work(s) for s, o, k in zip(shapes, owner, w) if o == r and k == j) for j in range(waves)]
                mine = [ns_work(s) for s, o in zip(shapes, owner) if o == r]
                if mine:
                    assert max(load) - min(load) <= max(mine)


SHAPES3 = [(24, 40), (8, 64)]


def exact_grads(rank, step):
    # small integer multiples of 2^-12: every partial sum over ranks is exact in
    # fp32, whatever order the all-reduce adds them in
    g = torch.Generator().manual_seed(500 * rank + step)
    return [torch.randint(-512, 513, s, generator=g).float() * 2.0 ** -12 for s in SHAPES3]


def _worker3(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        opt = DistributedMuon(SHAPES3, local_step=oracle_local_step, device="cpu")
        g = torch.Generator().manual_seed(3)
        Ws = [torch.randn(s, generator=g) * 0.02 for s in SHAPES3]
        rms = None
        for t in range(STEPS):
            rms = opt.step(list(zip(Ws, exact_grads(rank, t))), lr=LR, weight_decay=WD, momentum=MU).clone()
        out.put((rank, [W.numpy().copy() for W in Ws], rms.numpy().copy(), sorted(opt.M), opt.owner))
    finally:
        dist.destroy_process_group()


def test_three_ranks_with_an_idle_owner():
    # two matrices on three ranks: one rank owns nothing, but still joins every
    # collective and ends with the same weights
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker3, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    g = torch.Generator().manual_seed(3)
    Ws = [torch.randn(s, generator=g) * 0.02 for s in SHAPES3]
    Ms = [torch.zeros(s) for s in SHAPES3]
    for t in range(STEPS):
        Gsum = [sum(gs) for gs in zip(*(exact_grads(r, t) for r in range(world)))]
        ref_rms = oracle_local_step(list(zip(Ws, Gsum, Ms)), lr=LR, weight_decay=WD, momentum=MU)
    owners = res[0][4]
    assert len(set(owners)) == 2                       # one of the three ranks is idle
    for rank, W_out, rms, owned, owner in res:
        assert owner == owners
        for a, b in zip(W_out, Ws):
            assert np.array_equal(a, b.numpy())
        assert np.array_equal(rms, ref_rms.numpy())
        assert owned == [i for i, r in enumerate(owner) if r == rank]
