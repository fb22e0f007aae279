"""Owner-computes sharding of the Muon step over torch.distributed ranks.

Each hidden matrix is an independent unit of the step.  muon_partition (C
ABI, host only) gives every matrix one owner rank; the owner alone keeps its
momentum buffer and runs its step (through the library on the GPU); the
updated weights then travel from each owner to every other rank.  Only
plumbing lives here: the partition is the library's and the step is the
library's; torch.distributed moves the bytes (NCCL on GPUs, gloo on CPUs).

Layout.  The weights are re-pointed (Tensor.set_) into flat buffers, one per
(owner, stage): stage s of owner r holds, back to back, the s-th of `stages`
cost-balanced slices of r's matrices.  An owner's stage therefore leaves in
one broadcast straight from the weights' own storage, and lands in the same
place on every other rank, with no gather or scatter copy.

Overlap.  A step runs the owned matrices stage by stage.  As soon as stage s
is enqueued, the broadcasts of stage s (one per owner, in rank order, the
same sequence on every rank) are issued asynchronously; with NCCL they run on
the communicator's stream after the compute stream's work up to that point,
so the exchange of stage s overlaps the Newton-Schulz of stage s + 1.  The
step waits for all of them before it returns.
"""

from __future__ import annotations

from typing import Callable, List, Optional, Sequence

from .binding import partition


def _as_matrix(shape) -> tuple:
    """rows x cols of a weight stepped as a matrix (trailing dims flattened)."""
    cols = 1
    for d in shape[1:]:
        cols *= int(d)
    return int(shape[0]), cols


def _nominal_cost(rows: int, cols: int) -> float:
    """The cost muon_partition balances: 5 (4 m^2 n + 2 m^3) + 5600 rows cols."""
    m, n = min(rows, cols), max(rows, cols)
    return 5.0 * (4.0 * m * m * n + 2.0 * m ** 3) + 5600.0 * rows * cols


def _contiguous_strides(shape) -> tuple:
    out, acc = [], 1
    for d in reversed(shape):
        out.append(acc)
        acc *= int(d)
    return tuple(reversed(out))


def split_stages(idx: Sequence[int], costs: Sequence[float], stages: int) -> List[List[int]]:
    """Cut the ordered list `idx` into `stages` consecutive slices of about
    equal total cost (some may be empty); deterministic."""
    total = sum(costs[i] for i in idx)
    out: List[List[int]] = [[] for _ in range(max(1, stages))]
    acc = 0.0
    for i in idx:
        s = min(len(out) - 1, int(acc * len(out) / total)) if total > 0 else 0
        out[s].append(i)
        acc += costs[i]
    return out


class ShardedMuon:
    """weights: every rank's full list of hidden weights (same shapes, dtype
    and order on all ranks, one device); they are moved into the sharded
    flat storage in place (their values are kept).  momentum: buffers for the
    matrices this rank owns (create them from `owned`), None elsewhere.
    local_step(idx, grads, momentum): runs the Muon step on the owned
    matrices idx (default: one MuonContext.step over groups of equal shape).
    stages: slices per owner whose exchange overlaps the next slice's step."""

    def __init__(self, weights: Sequence, group=None, ctx=None, hp=None,
                 local_step: Optional[Callable] = None, stages: int = 2):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.weights = list(weights)
        mats = [_as_matrix(tuple(w.shape)) for w in self.weights]
        self.owner = partition(mats, self.world)
        self.owned = [i for i, o in enumerate(self.owner) if o == self.rank]
        self.ctx = ctx
        self.hp = hp
        self.local_step = local_step
        self.stages = max(1, int(stages))
        costs = [_nominal_cost(r, c) for r, c in mats]
        # stage_idx[r][s]: matrices of owner r in its stage s
        self.stage_idx = [split_stages([i for i, o in enumerate(self.owner) if o == r], costs, self.stages)
                          for r in range(self.world)]
        self.trace: List[tuple] = []
        self._flat = self._adopt_flat_storage()

    def by_rank(self) -> List[List[int]]:
        out = [[] for _ in range(self.world)]
        for i, o in enumerate(self.owner):
            out[o].append(i)
        return out

    def _adopt_flat_storage(self):
        """One flat buffer per (owner, stage); every weight is copied into its
        slot and re-pointed there."""
        import torch
        flat = []
        for r in range(self.world):
            row = []
            for idx in self.stage_idx[r]:
                if not idx:
                    row.append(None)
                    continue
                ws = [self.weights[i] for i in idx]
                buf = torch.empty(sum(w.numel() for w in ws), dtype=ws[0].dtype, device=ws[0].device)
                off = 0
                with torch.no_grad():
                    for w in ws:
                        n = w.numel()
                        buf[off:off + n].copy_(w.reshape(-1))
                        w.set_(buf.untyped_storage(), off, w.shape, _contiguous_strides(w.shape))
                        off += n
                row.append(buf)
            flat.append(row)
        return flat

    def _local(self, idx, grads, momentum, stream):
        if not idx:
            return
        if self.local_step is not None:
            self.local_step(idx, grads, momentum)
            return
        groups = {}
        for i in idx:
            groups.setdefault(tuple(self.weights[i].shape), []).append(i)
        self.ctx.step([dict(weights=[self.weights[i] for i in ix], grads=[grads[i] for i in ix],
                            momentum=[momentum[i] for i in ix]) for ix in groups.values()],
                      self.hp, stream)

    def step(self, grads: Sequence, momentum: Sequence, stream=None):
        """grads: full list (only owned entries are read); momentum: full
        list, None for matrices owned elsewhere.  stream: the CUDA stream of
        the step (default: the current one); the broadcasts are ordered
        after the work enqueued on it."""
        import contextlib

        import torch
        scope = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
        with scope:
            self.trace = []
            works = []
            for s in range(self.stages):
                self._local(self.stage_idx[self.rank][s], grads, momentum, stream)
                self.trace.append(("step", self.rank, s))
                works += self._issue(s)
            for w in works:
                w.wait()

    def _issue(self, s):
        """Broadcasts of stage s, one per owner that has matrices in it."""
        works = []
        for r in range(self.world):
            buf = self._flat[r][s]
            if buf is None:
                continue
            works.append(self.dist.broadcast(buf, src=r, group=self.group, async_op=True))
            self.trace.append(("send", r, s))
        return works

    def exchange(self):
        """Every stage of every owner, without a local step (blocking)."""
        works = []
        for s in range(self.stages):
            works += self._issue(s)
        for w in works:
            w.wait()
