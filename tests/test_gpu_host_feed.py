"""MuonStep.step_from_host: gradients in pinned host memory, copied on a side stream.

The copy overlaps the previous step's kernels, but every step must see exactly its own
gradients: the parameters and momenta must equal, bit for bit, those of the same steps
taken with the gradients already on the device.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from muon_newton_schulz_07_b200 import binding as B
from muon_newton_schulz_07_b200.optimizer import MuonStep

pytestmark = pytest.mark.gpu

SHAPES = [(256, 256), (512, 1024), (1024, 512), (384, 640)]


def test_host_fed_steps_equal_device_fed_steps():
    torch.manual_seed(5)
    dev = torch.device("cuda")
    W0 = [(torch.randn(s, device=dev) * 0.02).to(torch.bfloat16) for s in SHAPES]
    M0 = [(torch.randn(s, device=dev) * 1e-3).to(torch.bfloat16) for s in SHAPES]
    steps = 5
    G = [[(torch.randn(s, device=dev) * 1e-3).to(torch.bfloat16) for s in SHAPES] for _ in range(steps)]
    G_host = [[g.cpu().pin_memory() for g in gs] for gs in G]

    Wa, Ma = [w.clone() for w in W0], [m.clone() for m in M0]
    Wb, Mb = [w.clone() for w in W0], [m.clone() for m in M0]
    a = MuonStep(SHAPES)
    b = MuonStep(SHAPES)
    for i in range(steps):
        a(Wa, G[i], Ma, lr=0.02, beta=0.95, weight_decay=0.1)
        b.step_from_host(Wb, G_host[i], Mb, lr=0.02, beta=0.95, weight_decay=0.1)
    torch.cuda.synchronize()
    assert a.status() == B.MUON_OK and b.status() == B.MUON_OK
    for wa, wb, ma, mb in zip(Wa, Wb, Ma, Mb):
        assert torch.equal(wa, wb)
        assert torch.equal(ma, mb)
    assert not all(torch.equal(w0, wa) for w0, wa in zip(W0, Wa))


def test_host_fed_rejects_mismatched_gradients():
    op = MuonStep(SHAPES)
    W = [torch.zeros(s, device="cuda", dtype=torch.bfloat16) for s in SHAPES]
    M = [torch.zeros(s, device="cuda", dtype=torch.bfloat16) for s in SHAPES]
    bad = [torch.zeros(s, dtype=torch.bfloat16).pin_memory() for s in SHAPES[:-1]]
    with pytest.raises(ValueError):
        op.step_from_host(W, bad, M)
    wrong = [torch.zeros((s[1], s[0]), dtype=torch.bfloat16).pin_memory() for s in SHAPES]
    with pytest.raises(ValueError):
        op.step_from_host(W, wrong, M)
    np.testing.assert_array_equal(torch.stack([w.float().abs().sum() for w in W]).cpu().numpy(), 0.0)


def test_step_replays_from_a_cuda_graph():
    # muon_step enqueues kernels and one memset on the caller's stream and never synchronises,
    # so a captured step replayed twice must equal two eager steps bit for bit.
    torch.manual_seed(6)
    dev = torch.device("cuda")
    W0 = [(torch.randn(s, device=dev) * 0.02).to(torch.bfloat16) for s in SHAPES]
    M0 = [(torch.randn(s, device=dev) * 1e-3).to(torch.bfloat16) for s in SHAPES]
    G = [(torch.randn(s, device=dev) * 1e-3).to(torch.bfloat16) for s in SHAPES]
    We, Me = [w.clone() for w in W0], [m.clone() for m in M0]
    Wg, Mg = [w.clone() for w in W0], [m.clone() for m in M0]
    eager, graphed = MuonStep(SHAPES), MuonStep(SHAPES)
    for _ in range(2):
        eager(We, G, Me, lr=0.02, beta=0.95)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        graphed(Wg, G, Mg, lr=0.02, beta=0.95, stream=s)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert eager.status() == B.MUON_OK and graphed.status() == B.MUON_OK
    for we, wg, me, mg in zip(We, Wg, Me, Mg):
        assert torch.equal(we, wg)
        assert torch.equal(me, mg)
