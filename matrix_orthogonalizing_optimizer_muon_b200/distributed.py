"""Data-parallel Muon over torch.distributed.

"Muon is Scalable for LLM Training" (Sec. 2.3, Algorithm 1, "Distributed
Muon") keeps ZeRO-1's partitioned optimizer state.  Its steps are:
- reduce-scatter the gradients;
- apply momentum on each rank's shard;
- gather the full matrices (bf16) on every rank;
- run Newton-Schulz on each gathered matrix, keeping only the rank's own slice;
- all-gather the updated parameters.

Here the unit of partition is a whole matrix rather than a flat slice.  Every
matrix has one owner rank (a greedy longest-first assignment balanced by
Newton-Schulz FLOPs), which holds its momentum and runs its Newton-Schulz
step.  One step is:
  1. reduce the gradients to their owners: one reduce-scatter over a flat
     buffer laid out owner by owner;
  2. on each owner, the full Muon step of its matrices (libmuon's kernels);
  3. all-gather the owners' updated weights (and update RMS values).
So Newton-Schulz never runs twice and the gather of step 6 of the algorithm
disappears: a matrix's gradient is already whole on its owner.  The
optimizer state is still partitioned as in ZeRO-1.  Communication per step
is one reduce-scatter of the fp32 gradients and one all-gather of the fp32
weights, the "4 + 4" of the pages' Distributed AdamW comparison.

The gradients are summed, not averaged.  The orthogonalised update is
invariant to a common scale of M and G, so the weights move exactly as with
the average.  Only the stored momentum, and the logged RMS of O, which is
itself scale free, see the difference.

The collectives are torch.distributed's (NCCL on GPUs).  Packing tensors into
the flat buffers is plain device copies; every step of the method runs in
libmuon.  Backends without reduce-scatter (gloo) use an all-reduce and keep
the owner's part.
"""

from __future__ import annotations

from typing import Callable, Sequence

import torch
import torch.distributed as dist


def ns_work(shape) -> float:
    """Newton-Schulz FLOPs of one matrix per iteration (symmetry-aware count)."""
    m, n = min(shape), max(shape)
    return float(m * (m + 1) * n + m * m * (m + 1) + 2 * m * m * n)


def assign_owners(shapes: Sequence[tuple], world: int) -> list[int]:
    """Greedy longest-processing-time assignment of matrices to ranks by
    Newton-Schulz work; ties go to the lowest rank, so every rank computes the
    same answer."""
    order = sorted(range(len(shapes)), key=lambda i: (-ns_work(shapes[i]), i))
    load = [0.0] * world
    owner = [0] * len(shapes)
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        owner[i] = r
        load[r] += ns_work(shapes[i])
    return owner


class DistributedMuon:
    """Muon over the ranks of `group`: call `step` on every rank with that
    rank's full-model (W, G) list; W ends equal on all ranks.

    `local_step(params, M_list, **hp)` runs the Muon step of the owned
    matrices in place (params = [(W, G, M), ...]); it defaults to a libmuon
    `MuonPlan` on the current CUDA device."""

    def __init__(self, shapes, *, group=None, local_step: Callable | None = None, device=None):
        self.shapes = [tuple(int(v) for v in s) for s in shapes]
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.owner = assign_owners(self.shapes, self.world)
        self.owned = [i for i, r in enumerate(self.owner) if r == self.rank]
        sizes = [s[0] * s[1] for s in self.shapes]
        # flat layout: rank 0's matrices, then rank 1's, ...; each rank's part padded to `chunk`
        self.offsets, per_rank = {}, [0] * self.world
        for i in range(len(self.shapes)):
            r = self.owner[i]
            self.offsets[i] = per_rank[r]
            per_rank[r] += sizes[i]
        self.chunk = max(1, max(per_rank))
        self.device = torch.device(device) if device is not None else (
            torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else torch.device("cpu"))
        self.M = {i: torch.zeros(self.shapes[i], device=self.device) for i in self.owned}
        self.send = torch.empty(self.world * self.chunk, device=self.device)
        self.mine = torch.empty(self.chunk, device=self.device)
        self.gathered = torch.empty(self.world * self.chunk, device=self.device)
        self.rms = torch.zeros(len(self.shapes), device=self.device)
        self._local_step = local_step
        self._plan = None
        backend = dist.get_backend(group)
        self._has_rs = backend == "nccl"

    def _view(self, flat, rank, i):
        o = rank * self.chunk + self.offsets[i]
        r, c = self.shapes[i]
        return flat[o:o + r * c].view(r, c)

    def _default_step(self, params, **hp):
        from .api import MuonPlan
        if self._plan is None:
            self._plan = MuonPlan([self.shapes[i] for i in self.owned])
        rms = torch.zeros(len(params), device=self.device)
        self._plan.step(params, update_rms=rms, **hp)
        return rms

    def step(self, params, **hp) -> torch.Tensor:
        """One data-parallel Muon step.  params: [(W, G), ...] for every
        matrix, on every rank (W fp32, G fp32 or bf16).  Returns the update
        RMS of every matrix (fp32, identical on all ranks)."""
        if len(params) != len(self.shapes):
            raise ValueError("one (W, G) per matrix")
        # 1. gradients to their owners (summed over ranks)
        for i, (_, G) in enumerate(params):
            self._view(self.send, self.owner[i], i).copy_(G)
        if self._has_rs:
            dist.reduce_scatter_tensor(self.mine, self.send, op=dist.ReduceOp.SUM, group=self.group)
        else:
            dist.all_reduce(self.send, op=dist.ReduceOp.SUM, group=self.group)
            self.mine.copy_(self.send[self.rank * self.chunk:(self.rank + 1) * self.chunk])
        # 2. the owner's Muon step on its matrices
        local = []
        for i in self.owned:
            r, c = self.shapes[i]
            o = self.offsets[i]
            local.append((params[i][0], self.mine[o:o + r * c].view(r, c), self.M[i]))
        self.rms.zero_()
        if local:
            step = self._local_step if self._local_step is not None else self._default_step
            rms_owned = step(local, **hp)
            for k, i in enumerate(self.owned):
                self.rms[i] = rms_owned[k]
        # 3. updated weights (and RMS values) from their owners to every rank
        for i in self.owned:
            r, c = self.shapes[i]
            o = self.offsets[i]
            self.mine[o:o + r * c].view(r, c).copy_(params[i][0])
        dist.all_gather_into_tensor(self.gathered, self.mine, group=self.group)
        for i, (W, _) in enumerate(params):
            if self.owner[i] != self.rank:
                W.copy_(self._view(self.gathered, self.owner[i], i))
        dist.all_reduce(self.rms, op=dist.ReduceOp.SUM, group=self.group)
        return self.rms

    def close(self) -> None:
        if self._plan is not None:
            self._plan.close()
            self._plan = None
