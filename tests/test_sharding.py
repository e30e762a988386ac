"""Multi-rank path on CPU: ownership by matrix, and the sharded step (world size 2, gloo).

The per-rank step is injected: here the float64 oracle steps the owned matrices, so the test checks
the sharding and the exchange (not the kernels) against the unsharded oracle over the whole set.
"""
from __future__ import annotations

import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from muon_newton_schulz_07_b200 import inputs as I
from muon_newton_schulz_07_b200.sharding import ShardedMuon, loads, partition


@pytest.mark.parametrize("world", [1, 2, 4, 8])
@pytest.mark.parametrize("name", ["d24", "l38b", "gpt2s"])
def test_partition_covers_every_matrix_once_and_balances(name, world):
    shapes = I.WORKLOADS[name].shapes
    owner = partition(shapes, world)
    assert len(owner) == len(shapes) and set(owner) <= set(range(world))
    ld = loads(shapes, owner, world)
    # greedy LPT: the heaviest rank exceeds the mean by at most the largest single matrix
    from muon_newton_schulz_07_b200.sharding import matrix_cost

    biggest = max(matrix_cost(*s) for s in shapes)
    assert max(ld) <= sum(ld) / world + biggest
    if name == "d24" and world <= 8:
        assert max(ld) / (sum(ld) / world) < 1.10


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SHAPES = [(32, 48), (48, 32), (40, 40), (16, 64), (64, 16), (24, 24), (8, 8)]
HP = dict(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7, nesterov=True, ns_steps=5)


def _oracle_local_step(W, G, M, lr, beta, weight_decay, eps, nesterov, ns_steps):
    hp = O.Hyper(lr=lr, beta=beta, weight_decay=weight_decay, eps=eps, nesterov=nesterov, ns_steps=ns_steps)
    for w, g, m in zip(W, G, M):
        w1, m1, _ = O.muon_step(w.numpy(), g.numpy(), m.numpy(), hp)
        w.copy_(torch.from_numpy(w1))
        m.copy_(torch.from_numpy(m1))


def _inputs():
    rng = np.random.default_rng(30)
    W = [torch.from_numpy(rng.standard_normal(s)) for s in SHAPES]
    G = [torch.from_numpy(rng.standard_normal(s)) for s in SHAPES]
    M = [torch.from_numpy(rng.standard_normal(s)) for s in SHAPES]
    return W, G, M


def _worker(rank, world, port, outdir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        W, G, M = _inputs()
        sh = ShardedMuon(SHAPES, rank, world, local_step=_oracle_local_step)
        M_owned = [M[i] for i in sh.owned]
        sh.step(W, G, M_owned, **HP)
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), *[w.numpy() for w in W], owned=np.array(sh.owned),
                 **{f"m{i}": M[i].numpy() for i in sh.owned})
    finally:
        dist.destroy_process_group()


def test_sharded_step_equals_unsharded_world2():
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(world, _free_port(), d), nprocs=world, join=True, start_method="spawn")
        W, G, M = _inputs()
        hp = O.Hyper(**{k: v for k, v in HP.items()})
        ref = [O.muon_step(w.numpy(), g.numpy(), m.numpy(), hp) for w, g, m in zip(W, G, M)]
        owned_all = []
        for r in range(world):
            z = np.load(os.path.join(d, f"rank{r}.npz"))
            for i in range(len(SHAPES)):
                # every rank ends with every matrix's updated parameters, bit for bit
                assert np.array_equal(z[f"arr_{i}"], ref[i][0]), (r, i)
            for i in z["owned"]:
                assert np.array_equal(z[f"m{i}"], ref[i][1])
            owned_all += list(z["owned"])
        assert sorted(owned_all) == list(range(len(SHAPES)))


def _local_grad(rank, G):
    # each rank's own gradient: the shared part plus a rank-dependent part
    rng = np.random.default_rng(100 + rank)
    return [g + torch.from_numpy(rng.standard_normal(tuple(g.shape))) for g in G]


def _worker_local_grads(rank, world, port, outdir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        W, G, M = _inputs()
        sh = ShardedMuon(SHAPES, rank, world, local_step=_oracle_local_step)
        M_owned = [M[i] for i in sh.owned]
        sh.step_local_grads(W, _local_grad(rank, G), M_owned, **HP)
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), *[w.numpy() for w in W], owned=np.array(sh.owned),
                 **{f"m{i}": M[i].numpy() for i in sh.owned})
    finally:
        dist.destroy_process_group()


def test_reduce_scatter_step_equals_unsharded_step_on_the_mean_gradient():
    # Each rank brings its own gradients; the sharded step averages them by a reduce-scatter over
    # the ownership, steps its own matrices and all-gathers W.  The result must be the unsharded
    # step on the mean gradient, bit for bit (two float64 summands: the sum and the halving are exact).
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker_local_grads, args=(world, _free_port(), d), nprocs=world, join=True,
                           start_method="spawn")
        W, G, M = _inputs()
        locals_ = [_local_grad(r, G) for r in range(world)]
        G_mean = [(a + b) / 2 for a, b in zip(*locals_)]
        hp = O.Hyper(**{k: v for k, v in HP.items()})
        ref = [O.muon_step(w.numpy(), g.numpy(), m.numpy(), hp) for w, g, m in zip(W, G_mean, M)]
        owned_all = []
        for r in range(world):
            z = np.load(os.path.join(d, f"rank{r}.npz"))
            for i in range(len(SHAPES)):
                assert np.array_equal(z[f"arr_{i}"], ref[i][0]), (r, i)
            for i in z["owned"]:
                assert np.array_equal(z[f"m{i}"], ref[i][1])
            owned_all += list(z["owned"])
        assert sorted(owned_all) == list(range(len(SHAPES)))
