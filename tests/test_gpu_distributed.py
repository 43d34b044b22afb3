"""Data-parallel Muon with its default local step (libmuon on the GPU) over a
one-rank NCCL group, in two waves: the packing kernels, the asynchronous
reduce-scatter / all-gather per wave and the owner step all run on the
device.  Every matrix of every step is compared with the fp64 oracle run from
the GPU's own previous weights and momentum (the reduction of one rank is the
identity and an fp32 copy of a bf16 gradient is exact); the result must also
equal a plain MuonPlan step bit for bit."""

import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan, PackPlan
from matrix_orthogonalizing_optimizer_muon_b200.distributed import DistributedMuon

from _gpu import ABC32, LR, MU, WD, check_step, host64

pytestmark = pytest.mark.gpu

SHAPES = [(256, 128), (300, 520), (520, 300), (1408, 2048), (2048, 1408), (33, 17), (2048, 64)]


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_matches_the_oracle_and_the_plan():
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        g = torch.Generator(device="cuda")
        g.manual_seed(21)
        Ws = [torch.randn(s, device="cuda", generator=g) * 0.02 for s in SHAPES]
        W2 = [W.clone() for W in Ws]
        M2 = [torch.zeros(s, device="cuda") for s in SHAPES]
        opt = DistributedMuon(SHAPES, waves=2)
        assert sorted(opt.owned) == list(range(len(SHAPES)))
        assert all(len(w) > 0 for w in opt.owned_in)
        plan = MuonPlan(SHAPES)
        rms2 = torch.zeros(len(SHAPES), device="cuda")
        hp = dict(lr=LR, weight_decay=WD, momentum=MU, coeffs=ABC32)
        for t in range(3):
            Gs = [(torch.randn(s, device="cuda", generator=g) * 1e-3).to(torch.bfloat16) for s in SHAPES]
            before = [(host64(W), host64(opt.M[i]), host64(G)) for i, (W, G) in enumerate(zip(Ws, Gs))]
            rms1 = opt.step(list(zip(Ws, Gs)), **hp)
            torch.cuda.synchronize()
            for i in range(len(SHAPES)):
                W0, M0, G0 = before[i]
                check_step(W0, M0, G0, host64(Ws[i]), host64(opt.M[i]), float(rms1[i]), lr=LR, wd=WD, mu=MU)
            plan.step(list(zip(W2, Gs, M2)), update_rms=rms2, **hp)
        torch.cuda.synchronize()
        for a, b in zip(Ws, W2):
            assert torch.equal(a, b)
        assert torch.equal(rms1, rms2)
        opt.close()
        plan.close()
    finally:
        dist.destroy_process_group()


def test_pack_plan_copies_and_converts_every_segment():
    g = torch.Generator(device="cuda")
    g.manual_seed(22)
    # ragged sizes across the 64 Ki-element chunks, misaligned views, both conversions
    base = torch.randn(300000, device="cuda", generator=g)
    srcs = [base[:1], base[3:3 + 70001], base[80000:80000 + 65536].to(torch.bfloat16), base[200000:200100]]
    dst_flat = torch.full((140000,), float("nan"), device="cuda")
    dsts = [dst_flat[:1], dst_flat[5:5 + 70001], dst_flat[70010:70010 + 65536],
            torch.empty(100, device="cuda", dtype=torch.bfloat16)]
    plan = PackPlan(list(zip(srcs, dsts)))
    plan.run()
    torch.cuda.synchronize()
    for s, d in zip(srcs, dsts):
        assert torch.equal(d, s.to(d.dtype))  # fp32 -> bf16 rounds to nearest even, as torch does
    # destinations that overlap, or a source that overlaps a destination, are refused
    from matrix_orthogonalizing_optimizer_muon_b200 import _lib as L
    with pytest.raises(L.MuonError) as e:
        PackPlan([(srcs[1], dst_flat[:70001]), (srcs[0], dst_flat[10:11])])
    assert e.value.status == L.MUON_ERR_ALIAS
    with pytest.raises(L.MuonError) as e:
        PackPlan([(base[:100], base[50:150])])
    assert e.value.status == L.MUON_ERR_ALIAS
    plan.close()
