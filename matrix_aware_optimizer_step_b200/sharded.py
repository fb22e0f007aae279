"""Owner-computes sharding of the Muon step over torch.distributed ranks.

Each hidden matrix is an independent unit of the step.  muon_partition (C
ABI, host only) gives every matrix one owner rank; the owner alone keeps its
momentum buffer and runs its step (through the library on the GPU); then
every owner sends its updated weights to the other ranks, one broadcast per
owner of a flat buffer of its matrices.  Only plumbing lives here: the
partition is the library's and the step is the library's; torch.distributed
moves the bytes (NCCL on GPUs, gloo on CPUs).
"""

from __future__ import annotations

from typing import Callable, List, Optional, Sequence

from .binding import partition


class ShardedMuon:
    """weights: every rank's full list of hidden weights (same shapes and
    order on all ranks).  momentum: buffers for the matrices this rank owns
    (created by the caller from `owned`), None elsewhere.  local_step(idx,
    grads_by_idx): runs the Muon step on this rank's owned matrices (default:
    a MuonContext.step over groups of equal shape)."""

    def __init__(self, weights: Sequence, group=None, ctx=None, hp=None,
                 local_step: Optional[Callable] = None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.weights = list(weights)
        self.owner = partition([tuple(w.shape) for w in self.weights], self.world)
        self.owned = [i for i, o in enumerate(self.owner) if o == self.rank]
        self.ctx = ctx
        self.hp = hp
        self.local_step = local_step

    def by_rank(self) -> List[List[int]]:
        out = [[] for _ in range(self.world)]
        for i, o in enumerate(self.owner):
            out[o].append(i)
        return out

    def step(self, grads: Sequence, momentum: Sequence, stream=None):
        """grads: full list (only owned entries are read); momentum: full
        list, None for matrices owned elsewhere."""
        if self.local_step is not None:
            self.local_step(self.owned, grads, momentum)
        else:
            groups = {}
            for i in self.owned:
                groups.setdefault(tuple(self.weights[i].shape), []).append(i)
            self.ctx.step([dict(weights=[self.weights[i] for i in ix], grads=[grads[i] for i in ix],
                                momentum=[momentum[i] for i in ix]) for ix in groups.values()],
                          self.hp, stream)
        self.exchange()

    def exchange(self):
        """Owner r broadcasts the flat concatenation of its matrices."""
        import torch
        for r, idx in enumerate(self.by_rank()):
            if not idx:
                continue
            ws = [self.weights[i] for i in idx]
            if r == self.rank:
                flat = torch.cat([w.reshape(-1) for w in ws])
            else:
                flat = torch.empty(sum(w.numel() for w in ws), dtype=ws[0].dtype, device=ws[0].device)
            self.dist.broadcast(flat, src=r, group=self.group)
            if r != self.rank:
                off = 0
                for w in ws:
                    w.copy_(flat[off:off + w.numel()].view_as(w))
                    off += w.numel()
