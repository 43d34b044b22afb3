"""Data-parallel Muon over torch.distributed.

"Muon is Scalable for LLM Training" (Sec. 2.3, Algorithm 1, "Distributed
Muon") keeps ZeRO-1's partitioned optimizer state.  Its steps are:
- reduce-scatter the gradients;
- apply momentum on each rank's shard;
- gather the full matrices (bf16) on every rank;
- run Newton-Schulz on each gathered matrix, keeping only the rank's own slice;
- all-gather the updated parameters.
The same section notes that the gather's latency can be hidden by overlapping
it with computation.

Here the unit of partition is a whole matrix rather than a flat slice.  Every
matrix has one owner rank (a greedy longest-first assignment balanced by
Newton-Schulz FLOPs), which holds its momentum and runs its Newton-Schulz
step.  So Newton-Schulz never runs twice and the bf16 gather disappears: a
matrix's gradient is already whole on its owner.  The optimizer state is still
partitioned as in ZeRO-1, and the communication per step is one fp32
reduce-scatter of the gradients and one fp32 all-gather of the weights, the
"4 + 4" bytes per element of the pages' Distributed AdamW comparison.

Overlap.  Each rank's matrices are split into `waves` groups of about equal
Newton-Schulz work, and the flat buffers are laid out wave by wave (within a
wave, rank by rank).  One step is then
  1. pack every gradient into the flat buffer (one launch), and enqueue the
     reduce-scatter of every wave on the communication stream;
  2. for each wave k: wait for its reduce-scatter, run the owner's Muon step
     of its matrices (libmuon's kernels), pack its updated weights (one
     launch) and enqueue its all-gather, which then runs while wave k + 1
     computes (and reduce-scatter k + 1 ran while wave k computed);
  3. for each wave: wait for its all-gather and unpack the other ranks'
     weights into place (one launch per wave); then one index scatter and
     one all-reduce place every matrix's update RMS on every rank.
The launch count of a step depends on the number of waves only, not on the
number of matrices.

The gradients are summed, not averaged.  The orthogonalised update is
invariant to a common scale of M and G, so the weights move exactly as with
the average.  Only the stored momentum, and the logged RMS of O, which is
itself scale free, see the difference.

The collectives are torch.distributed's (NCCL on GPUs, with its own data
plane).  Packing on the GPU is libmuon's one-launch segment copy; on the CPU
(gloo) it is plain tensor copies.  Backends without reduce-scatter (gloo) use
an all-reduce and keep the owner's part.
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


def assign_waves(shapes: Sequence[tuple], owner: Sequence[int], world: int, waves: int) -> list[int]:
    """Split each rank's matrices into `waves` groups of about equal work
    (longest first to the lightest wave); deterministic on every rank."""
    wave = [0] * len(shapes)
    for r in range(world):
        mine = sorted((i for i in range(len(shapes)) if owner[i] == r), key=lambda i: (-ns_work(shapes[i]), i))
        load = [0.0] * waves
        for i in mine:
            k = min(range(waves), key=lambda w: (load[w], w))
            wave[i] = k
            load[k] += ns_work(shapes[i])
    return wave


class _Packer:
    """Copies a fixed list of (src, dst) tensor pairs: one libmuon launch on
    CUDA, tensor copies on the CPU.  Rebuilt when a pointer changes."""

    def __init__(self):
        self._key = None
        self._plan = None
        self._pairs = []

    def run(self, pairs):
        if not pairs:
            return
        key = tuple((s.data_ptr(), d.data_ptr(), s.dtype, d.dtype, s.numel()) for s, d in pairs)
        if pairs[0][1].is_cuda:
            if key != self._key:
                from .api import PackPlan
                self.close()
                self._plan = PackPlan(pairs)
                self._key = key
            self._plan.run()
        else:
            for s, d in pairs:
                d.copy_(s.reshape(d.shape))

    def close(self):
        if self._plan is not None:
            self._plan.close()
            self._plan = None
            self._key = None


class DistributedMuon:
    """Muon over the ranks of `group`: call `step` on every rank with that
    rank's full-model (W, G) list; W ends equal on all ranks.

    `local_step(params, **hp)` runs the Muon step of the owned matrices of one
    wave in place (params = [(W, G, M), ...]) and returns their update RMS;
    it defaults to a libmuon `MuonPlan` per wave on the current CUDA device."""

    def __init__(self, shapes, *, group=None, local_step: Callable | None = None, device=None, waves: int = 2):
        self.shapes = [tuple(int(v) for v in s) for s in shapes]
        n = len(self.shapes)
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.waves = max(1, int(waves))
        self.owner = assign_owners(self.shapes, self.world)
        self.wave = assign_waves(self.shapes, self.owner, self.world, self.waves)
        self.owned = [i for i in range(n) if self.owner[i] == self.rank]
        self.owned_in = [[i for i in self.owned if self.wave[i] == k] for k in range(self.waves)]
        sizes = [s[0] * s[1] for s in self.shapes]
        # flat layout: wave 0 [rank 0 | rank 1 | ...], wave 1 [...], ...; a rank's part of wave k holds its
        # wave-k matrices in index order and is padded to chunk[k]
        self.offset = [0] * n
        part = [[0] * self.world for _ in range(self.waves)]
        for i in range(n):
            k, r = self.wave[i], self.owner[i]
            self.offset[i] = part[k][r]
            part[k][r] += sizes[i]
        self.chunk = [max(1, max(p)) for p in part]
        self.base = [0] * self.waves
        for k in range(1, self.waves):
            self.base[k] = self.base[k - 1] + self.world * self.chunk[k - 1]
        total = self.base[-1] + self.world * self.chunk[-1]
        self.device = torch.device(device) if device is not None else (
            torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else torch.device("cpu"))
        self.M = {i: torch.zeros(self.shapes[i], device=self.device) for i in self.owned}
        self.send = torch.empty(total, device=self.device)      # gradients, every rank's part
        self.gathered = torch.empty(total, device=self.device)  # updated weights, every rank's part
        self.g_own = [torch.empty(c, device=self.device) for c in self.chunk]  # my reduced gradients per wave
        self.w_own = [torch.empty(c, device=self.device) for c in self.chunk]  # my updated weights per wave
        self.rms = torch.zeros(n, device=self.device)
        self._owned_idx = [torch.tensor(ix, dtype=torch.long, device=self.device) for ix in self.owned_in]
        self._local_step = local_step
        self._plans = [None] * self.waves
        self._pack_g = _Packer()
        self._pack_w = [_Packer() for _ in range(self.waves)]
        self._unpack = [_Packer() for _ in range(self.waves)]
        self._has_rs = dist.get_backend(group) == "nccl"

    def _slot(self, flat, i):
        """View of matrix i in a flat every-rank buffer."""
        k = self.wave[i]
        o = self.base[k] + self.owner[i] * self.chunk[k] + self.offset[i]
        r, c = self.shapes[i]
        return flat[o:o + r * c].view(r, c)

    def _own(self, bufs, i):
        """View of owned matrix i in this rank's per-wave buffer."""
        r, c = self.shapes[i]
        o = self.offset[i]
        return bufs[self.wave[i]][o:o + r * c].view(r, c)

    def _region(self, flat, k):
        return flat[self.base[k]:self.base[k] + self.world * self.chunk[k]]

    def _default_step(self, k, params, **hp):
        from .api import MuonPlan
        if self._plans[k] is None:
            self._plans[k] = MuonPlan([self.shapes[i] for i in self.owned_in[k]])
        rms = torch.zeros(len(params), device=self.device)
        self._plans[k].step(params, update_rms=rms, **hp)
        return rms

    def step(self, params, **hp) -> torch.Tensor:
        """One data-parallel Muon step.  params: [(W, G), ...] for every
        matrix, on every rank (W fp32, G fp32 or bf16).  Returns the update
        RMS of every matrix (fp32, identical on all ranks)."""
        if len(params) != len(self.shapes):
            raise ValueError("one (W, G) per matrix")
        # 1. every gradient into its owner's slot, then the reduce-scatters of all waves
        self._pack_g.run([(G, self._slot(self.send, i)) for i, (_, G) in enumerate(params)])
        rs = []
        for k in range(self.waves):
            region = self._region(self.send, k)
            if self._has_rs:
                rs.append(dist.reduce_scatter_tensor(self.g_own[k], region, op=dist.ReduceOp.SUM, group=self.group,
                                                     async_op=True))
            else:
                rs.append(dist.all_reduce(region, op=dist.ReduceOp.SUM, group=self.group, async_op=True))
        # 2. wave by wave: the owner's step, then that wave's weight all-gather
        ag = []
        rms_parts = []
        for k in range(self.waves):
            rs[k].wait()
            if not self._has_rs:
                self.g_own[k].copy_(self._region(self.send, k)[self.rank * self.chunk[k]:(self.rank + 1) * self.chunk[k]])
            mine = self.owned_in[k]
            if mine:
                local = [(params[i][0], self._own(self.g_own, i), self.M[i]) for i in mine]
                if self._local_step is not None:
                    rms_parts.append(self._local_step(local, **hp))
                else:
                    rms_parts.append(self._default_step(k, local, **hp))
                self._pack_w[k].run([(params[i][0], self._own(self.w_own, i)) for i in mine])
            else:
                rms_parts.append(None)
            ag.append(dist.all_gather_into_tensor(self._region(self.gathered, k), self.w_own[k], group=self.group,
                                                  async_op=True))
        # 3. the other ranks' weights into place, the update RMS everywhere
        for k in range(self.waves):
            ag[k].wait()
            self._unpack[k].run([(self._slot(self.gathered, i), params[i][0]) for i in range(len(self.shapes))
                                 if self.wave[i] == k and self.owner[i] != self.rank])
        self.rms.zero_()
        for k in range(self.waves):
            if rms_parts[k] is not None:
                self.rms.index_copy_(0, self._owned_idx[k], torch.as_tensor(rms_parts[k], device=self.device,
                                                                            dtype=torch.float32))
        dist.all_reduce(self.rms, op=dist.ReduceOp.SUM, group=self.group)
        return self.rms

    def close(self) -> None:
        for k, p in enumerate(self._plans):
            if p is not None:
                p.close()
                self._plans[k] = None
        for pk in [self._pack_g, *self._pack_w, *self._unpack]:
            pk.close()
