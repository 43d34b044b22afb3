"""Programmatic dependent launch does not change any result: the same seeded
steps (a plan of mixed shapes, the split-K Gram path of a single long-K
matrix, and an entropy call) run in subprocesses under every MUON_PDL mask
(no kernel class, the tensor-core launches, the elementwise launches, both)
and must give bitwise the same weights, momenta, update RMS values and
Newton-Schulz outputs.  A kernel that read its predecessor's output before
its griddepcontrol.wait would race and, on some run, differ."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import hashlib, sys
import torch
sys.path.insert(0, ROOT)
from matrix_orthogonalizing_optimizer_muon_b200.api import MuonPlan, EntropyPlan
torch.cuda.set_device(0)
g = torch.Generator(device="cuda")
g.manual_seed(77)
shapes = [(2048, 1408), (1408, 2048), (300, 520), (520, 300), (2048, 64), (33, 17), (1024, 1024)]
Ws = [torch.randn(s, device="cuda", generator=g) * 0.02 for s in shapes]
Ms = [torch.zeros(s, device="cuda") for s in shapes]
plan = MuonPlan(shapes)
rms = torch.zeros(len(shapes), device="cuda")
h = hashlib.sha256()
for t in range(3):
    Gs = [(torch.randn(s, device="cuda", generator=g) * 1e-3).to(torch.bfloat16) for s in shapes]
    plan.step(list(zip(Ws, Gs, Ms)), lr=4.2e-4, weight_decay=0.1, momentum=0.95, update_rms=rms)
    torch.cuda.synchronize()
    h.update(rms.cpu().numpy().tobytes())
for W, M in zip(Ws, Ms):
    h.update(W.cpu().numpy().tobytes()); h.update(M.cpu().numpy().tobytes())
# one long-K matrix: the Gram product is split along K and reduced in a second kernel
x = (torch.randn((2048, 8192), device="cuda", generator=g)).to(torch.bfloat16)
o = torch.empty((2048, 8192), device="cuda")
single = MuonPlan([(2048, 8192)])
single.orthogonalize([x], [o])
torch.cuda.synchronize()
h.update(o.cpu().numpy().tobytes())
ent = EntropyPlan(shapes)
H = ent.compute(Ws)
torch.cuda.synchronize()
h.update(H.cpu().numpy().tobytes())
assert plan.status() == 0 and single.status() == 0
print(h.hexdigest())
"""


def test_every_launch_mask_gives_bitwise_the_same_results():
    digests = {}
    for mask in ("0", "1", "2", "3"):
        env = dict(os.environ, MUON_PDL=mask)
        out = subprocess.run([sys.executable, "-c", CHILD.replace("ROOT", repr(ROOT))], capture_output=True,
                             text=True, timeout=600, env=env, cwd=ROOT)
        assert out.returncode == 0, (mask, out.stderr[-2000:])
        digests[mask] = out.stdout.strip().splitlines()[-1]
    assert len(set(digests.values())) == 1, digests
