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
buffer and runs one all-gather (NCCL on GPUs, gloo in the CPU tests); the
gradient reduce-scatter sums bf16 gradients in fp32.
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

    Data layout of the exchanges: one flat buffer of world segments, segment q holding the
    matrices rank q owns, back to back in owned order, padded to the longest segment.  Matrix i
    sits at `offset[i]`.  Packing into and unpacking out of that buffer are multi-tensor copies
    (one launch each, whatever the number of matrices); a trainer that keeps its gradients in the
    views returned by gradient_views() skips the packing altogether.
    """

    def __init__(self, shapes, rank: int, world: int, local_step: Callable = None, group=None, ns_steps: int = 5,
                 dtype=torch.bfloat16, device=None):
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.rank, self.world, self.group = rank, world, group
        self.owner = partition(self.shapes, world, ns_steps)
        self.owned = [i for i, r in enumerate(self.owner) if r == rank]
        self.by_rank = [[i for i, r in enumerate(self.owner) if r == q] for q in range(world)]
        self.sizes = [sum(self.shapes[i][0] * self.shapes[i][1] for i in idx) for idx in self.by_rank]
        self.longest = max(self.sizes) if self.sizes else 0
        self.offset = [0] * len(self.shapes)
        for q in range(world):
            off = q * self.longest
            for i in self.by_rank[q]:
                self.offset[i] = off
                off += self.shapes[i][0] * self.shapes[i][1]
        self._bufs = {}
        if local_step is None:
            from .optimizer import MuonStep

            local_step = MuonStep([self.shapes[i] for i in self.owned], dtype=dtype, device=device)
        self.local_step = local_step

    # ------------------------------------------------------------ flat buffers
    def _buffer(self, name, numel, dtype, device):
        """A cached flat buffer, zero-filled when first made (the padding is never written)."""
        key = (name, dtype, str(device))
        buf = self._bufs.get(key)
        if buf is None or buf.numel() != numel:
            buf = torch.zeros(numel, dtype=dtype, device=device)
            self._bufs[key] = buf
        return buf

    def _views(self, flat, idx, base=0):
        return [flat[self.offset[i] - base:self.offset[i] - base + self.shapes[i][0] * self.shapes[i][1]]
                .view(self.shapes[i]) for i in idx]

    def gradient_views(self, dtype=torch.bfloat16, device=None):
        """Views, one per matrix in caller order, into the flat buffer reduce_gradients sends.  A
        trainer that writes its gradients there (e.g. as the parameters' .grad) sends them without
        any packing copy."""
        flat = self._buffer("grad_send", self.world * self.longest, dtype, device)
        return self._views(flat, range(len(self.shapes)))

    # ------------------------------------------------------------ steps
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

        Every rank's gradients sit in the flat send buffer (segment q: the matrices rank q owns);
        one reduce-scatter sums segment q onto rank q, which divides by the number of ranks and
        rounds once to the gradients' dtype.  bf16 and fp16 gradients are summed in fp32 (the send
        buffer is widened by one cast), so the mean carries a single rounding to bf16 instead of
        one per addition; fp32 and fp64 gradients are summed in their own type.  This is the
        collective that replaces a replicated trainer's all-reduce: each rank receives 1/N of the
        data.  The returned tensors are views of one buffer, valid until the next call.
        """
        if self.world == 1:
            return [G_local[i] for i in self.owned]
        ref = G_local[0]
        dt, dev = ref.dtype, ref.device
        send = self._buffer("grad_send", self.world * self.longest, dt, dev)
        views = self._views(send, range(len(self.shapes)))
        if any(g.data_ptr() != v.data_ptr() for g, v in zip(G_local, views)):
            torch._foreach_copy_(views, list(G_local))
        acc = torch.float32 if dt in (torch.bfloat16, torch.float16) else dt
        wire = send if acc == dt else self._buffer("grad_wire", send.numel(), acc, dev).copy_(send)
        recv = self._buffer("grad_recv", self.longest, acc, dev)
        dist.reduce_scatter_tensor(recv, wire, op=dist.ReduceOp.SUM, group=self.group)
        recv.div_(self.world)
        out = recv if acc == dt else self._buffer("grad_mean", self.longest, dt, dev).copy_(recv)
        return self._views(out, self.owned, base=self.rank * self.longest)

    def exchange(self, W):
        """Every rank gets the parameters its peers own: one all-gather of the packed segments
        (all_gather_into_tensor into the flat layout), unpacked by one multi-tensor copy."""
        if self.world == 1:
            return
        ref = W[0]
        dt, dev = ref.dtype, ref.device
        send = self._buffer("w_send", self.longest, dt, dev)
        if self.owned:
            torch._foreach_copy_(self._views(send, self.owned, base=self.rank * self.longest),
                                 [W[i] for i in self.owned])
        recv = self._buffer("w_recv", self.world * self.longest, dt, dev)
        dist.all_gather_into_tensor(recv, send, group=self.group)
        others = [i for i in range(len(self.shapes)) if self.owner[i] != self.rank]
        if others:
            torch._foreach_copy_([W[i] for i in others], self._views(recv, others))
