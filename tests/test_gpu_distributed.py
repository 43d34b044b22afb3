"""Data-parallel Muon with its default local step (libmuon on the GPU) over a
one-rank NCCL group: the collectives' code path runs on the device, and the
result must equal a plain MuonPlan step bit for bit (the reduction of one
rank is the identity and an fp32 copy of a bf16 gradient is exact)."""

import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan
from matrix_orthogonalizing_optimizer_muon_b200.distributed import DistributedMuon

from _gpu import ABC32, LR, MU, WD

pytestmark = pytest.mark.gpu

SHAPES = [(256, 128), (300, 520), (520, 300), (1408, 2048)]


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_matches_the_plan():
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        g = torch.Generator(device="cuda")
        g.manual_seed(21)
        Ws = [torch.randn(s, device="cuda", generator=g) * 0.02 for s in SHAPES]
        W2 = [W.clone() for W in Ws]
        M2 = [torch.zeros(s, device="cuda") for s in SHAPES]
        opt = DistributedMuon(SHAPES)
        plan = MuonPlan(SHAPES)
        rms2 = torch.zeros(len(SHAPES), device="cuda")
        hp = dict(lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
        for t in range(3):
            Gs = [(torch.randn(s, device="cuda", generator=g) * 1e-3).to(torch.bfloat16) for s in SHAPES]
            rms1 = opt.step(list(zip(Ws, Gs)), **hp)
            plan.step(list(zip(W2, Gs, M2)), update_rms=rms2, **hp)
        torch.cuda.synchronize()
        for a, b in zip(Ws, W2):
            assert torch.equal(a, b)
        assert torch.equal(rms1, rms2)
        opt.close()
        plan.close()
    finally:
        dist.destroy_process_group()
