"""Sharding the Muon step over data-parallel ranks (one process per GPU).

Every matrix's step is independent of the others, so the work splits by whole
matrices: each rank owns a subset, keeps the momentum buffers of only that
subset, steps only those matrices, and the updated parameters are then
exchanged so that every rank holds all of W again (the exchange a replicated
data-parallel trainer needs after its optimizer step; with a reduce-scatter of
the gradients by the same ownership it replaces the gradient all-reduce).

Ownership is decided by greedy longest-processing-time over the per-matrix
cost: Newton-Schulz work k (3 m^2 n + m^3) with m = min, n = max, plus a
bandwidth term for the momentum and parameter passes expressed in the same
units.  The exchange packs each rank's owned parameters into one contiguous
buffer and runs one all-gather (NCCL on GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

import heapq
from typing import Callable, List, Sequence, Tuple

import torch
import torch.distributed as dist

# Flops a B200 runs in the time it moves one byte at its tensor/HBM ridge point (~2.25e15 / 7.7e12).
_FLOP_PER_BYTE = 290.0


def matrix_cost(rows: int, cols: int, ns_steps: int = 5, elem_bytes: int = 2) -> float:
    m, n = min(rows, cols), max(rows, cols)
    flops = ns_steps * (3.0 * m * m * n + float(m) ** 3)
    bytes_moved = 14.0 * elem_bytes / 2 * rows * cols  # G, M, W and X passes of one step
    return flops + _FLOP_PER_BYTE * bytes_moved


def partition(shapes: Sequence[Tuple[int, int]], world: int, ns_steps: int = 5) -> List[int]:
    """owner[i] for each matrix: greedy LPT, heaviest matrices first, ties to the lowest rank."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(shapes)), key=lambda i: (-matrix_cost(*shapes[i], ns_steps), i))
    heap = [(0.0, r) for r in range(world)]
    heapq.heapify(heap)
    owner = [0] * len(shapes)
    for i in order:
        load, r = heapq.heappop(heap)
        owner[i] = r
        heapq.heappush(heap, (load + matrix_cost(*shapes[i], ns_steps), r))
    return owner


def loads(shapes, owner, world, ns_steps=5):
    out = [0.0] * world
    for s, r in zip(shapes, owner):
        out[r] += matrix_cost(*s, ns_steps)
    return out


class ShardedMuon:
    """Muon over a replicated parameter set, sharded by matrix across the ranks of `group`.

    local_step(W_owned, G_owned, M_owned) performs the Muon step on the owned matrices in place
    (by default a MuonStep over their shapes); W, G are the full lists on every rank and M holds
    only the owned momentum buffers, in owned order.
    """

    def __init__(self, shapes, rank: int, world: int, local_step: Callable = None, group=None, ns_steps: int = 5,
                 dtype=torch.bfloat16, device=None):
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.rank, self.world, self.group = rank, world, group
        self.owner = partition(self.shapes, world, ns_steps)
        self.owned = [i for i, r in enumerate(self.owner) if r == rank]
        self.by_rank = [[i for i, r in enumerate(self.owner) if r == q] for q in range(world)]
        self.sizes = [sum(self.shapes[i][0] * self.shapes[i][1] for i in idx) for idx in self.by_rank]
        if local_step is None:
            from .optimizer import MuonStep

            local_step = MuonStep([self.shapes[i] for i in self.owned], dtype=dtype, device=device)
        self.local_step = local_step

    def step(self, W, G, M_owned, **hp):
        """A step from gradients already averaged over the ranks (G: the full list on every rank)."""
        if self.owned:
            self.local_step([W[i] for i in self.owned], [G[i] for i in self.owned], M_owned, **hp)
        self.exchange(W)

    def step_local_grads(self, W, G_local, M_owned, **hp):
        """A data-parallel step from this rank's own gradients: average them over the ranks by a
        reduce-scatter that hands each rank only the matrices it owns, step those, all-gather W."""
        G_owned = self.reduce_gradients(G_local)
        if self.owned:
            self.local_step([W[i] for i in self.owned], G_owned, M_owned, **hp)
        self.exchange(W)

    def reduce_gradients(self, G_local):
        """The mean over the ranks of the owned matrices' gradients, in owned order.

        Every rank packs its full list of local gradients into one buffer, rank q's owned matrices
        in segment q (segments padded to the longest); one reduce-scatter sums segment q onto rank
        q, which divides by the number of ranks.  The sum runs in the gradients' dtype.  This is
        the collective that replaces a replicated trainer's all-reduce: each rank receives 1/N of
        the data instead of all of it.  The returned tensors are views of one fresh buffer.
        """
        if self.world == 1:
            return [G_local[i] for i in self.owned]
        ref = G_local[0]
        longest = max(self.sizes)
        send = torch.zeros(self.world * longest, dtype=ref.dtype, device=ref.device)
        for q in range(self.world):
            off = q * longest
            for i in self.by_rank[q]:
                n = G_local[i].numel()
                send[off:off + n].copy_(G_local[i].reshape(-1))
                off += n
        recv = torch.empty(longest, dtype=ref.dtype, device=ref.device)
        dist.reduce_scatter_tensor(recv, send, op=dist.ReduceOp.SUM, group=self.group)
        recv.div_(self.world)
        out, off = [], 0
        for i in self.owned:
            n = G_local[i].numel()
            out.append(recv[off:off + n].view_as(G_local[i]))
            off += n
        return out

    def exchange(self, W):
        """Every rank gets the parameters its peers own: one all-gather of packed, padded shards."""
        if self.world == 1:
            return
        ref = W[0]
        longest = max(self.sizes)
        send = torch.zeros(longest, dtype=ref.dtype, device=ref.device)
        if self.owned:
            torch.cat([W[i].reshape(-1) for i in self.owned], out=send[: self.sizes[self.rank]])
        recv = [torch.empty(longest, dtype=ref.dtype, device=ref.device) for _ in range(self.world)]
        dist.all_gather(recv, send, group=self.group)
        for q in range(self.world):
            if q == self.rank:
                continue
            off = 0
            for i in self.by_rank[q]:
                n = W[i].numel()
                W[i].copy_(recv[q][off:off + n].view_as(W[i]))
                off += n
