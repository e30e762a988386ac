"""The seeded synthetic inputs follow the recipe the design notes state (CPU only).

Shapes and counts of each workload, the distributions of W, G and M, determinism (the same
(workload, step, matrix, tensor) seeds give the same arrays, different ones do not), and the
structure of the stress set (orthonormal factors, singular values log-uniform in [1e-6, 1]).
"""
from __future__ import annotations

import numpy as np
import pytest

from muon_newton_schulz_07_b200 import inputs as I


def test_shapes_and_counts():
    d24 = I.WORKLOADS["d24"]
    assert len(d24.shapes) == 144 and I.param_count(d24) == 679_477_248
    assert d24.shapes.count((1536, 1536)) == 96 and d24.shapes.count((1536, 6144)) == 24
    assert d24.shapes.count((6144, 1536)) == 24
    gpt = I.WORKLOADS["gpt2s"]
    assert len(gpt.shapes) == 72 and gpt.shapes.count((768, 768)) == 48
    l38 = I.WORKLOADS["l38b"]
    assert len(l38.shapes) == 168 and I.param_count(l38) == 2_818_572_288
    st = I.WORKLOADS["stress"]
    assert len(st.shapes) == 256 and all(st.shapes.count(s) == 64 for s in set(st.shapes))
    s256 = I.WORKLOADS["single256"]
    assert s256.shapes == ((256, 256),) and s256.dtype == "f32"


def test_seeded_and_deterministic():
    wl = I.WORKLOADS["gpt2s"]
    a, b = I.gradient(wl, 3, 5), I.gradient(wl, 3, 5)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, I.gradient(wl, 4, 5))   # another step
    assert not np.array_equal(a[:768, :768], I.gradient(wl, 3, 0))  # another matrix
    assert not np.array_equal(I.weight(wl, 0), I.momentum(wl, 0))  # another tensor


def test_distributions():
    d24 = I.WORKLOADS["d24"]
    w = I.weight(d24, 0)
    assert w.dtype == np.float32 and abs(w.std() - 0.02) < 2e-4 and abs(w.mean()) < 1e-4
    assert not I.momentum(d24, 0).any()  # a fresh optimizer
    g = I.gradient(d24, 1, 0)
    row_std = g.std(axis=1)
    # row i ~ N(0, s_i^2), s_i = 10^U(-4, -2): the row scales span the two decades
    assert row_std.min() > 0.8e-4 and row_std.max() < 1.2e-2
    assert np.log10(row_std).max() - np.log10(row_std).min() > 1.8
    gpt = I.WORKLOADS["gpt2s"]
    gg = I.gradient(gpt, 1, 0)
    spikes = np.abs(gg) > 1e-3 * 20  # N(0, 1e-3^2) essentially never exceeds 20 sigma
    assert 0.007 < spikes.mean() < 0.013  # 1 % of the entries scaled by 100
    m = I.momentum(gpt, 0)
    assert abs(m.std() - 1e-3) < 2e-5
    one = I.WORKLOADS["single256"]
    assert abs(I.weight(one, 0).std() - 1.0) < 0.02


@pytest.mark.parametrize("idx", [0, 64, 128])
def test_stress_structure(idx):
    wl = I.WORKLOADS["stress"]
    r, c = wl.shapes[idx]
    P, s, Q = I.stress_factors(wl.wid, idx, r, c)
    k = min(r, c)
    assert np.allclose(P.T @ P, np.eye(k), atol=1e-10) and np.allclose(Q.T @ Q, np.eye(k), atol=1e-10)
    assert s.min() >= 1e-6 and s.max() <= 1.0
    # log-uniform: log10 s spreads evenly over [-6, 0]
    ls = np.log10(s)
    assert abs(ls.mean() + 3.0) < 0.25 and ls.min() < -5.5 and ls.max() > -0.5
    M = I.momentum(wl, idx)
    assert np.array_equal(I.gradient(wl, 1, idx), M)  # G = M, so the Nesterov blend is M
    sv = np.linalg.svd(M.astype(np.float64), compute_uv=False)
    assert np.allclose(np.sort(sv)[::-1][:8], np.sort(s)[::-1][:8], rtol=1e-5)


@pytest.mark.parametrize("idx", [0, 64, 128, 192])
def test_stress_structure_torch_generator(idx):
    # the device-side generator (used by the full-size GPU runs) follows the same recipe; run on
    # the CPU here: orthonormal factors, singular values exactly the log-uniform s
    import torch

    wl = I.WORKLOADS["stress"]
    r, c = wl.shapes[idx]
    M = I.stress_momentum_torch(wl, idx, "cpu")
    assert M.shape == (r, c) and M.dtype == torch.float32
    _, s, _ = I.stress_factors(wl.wid, idx, r, c)
    sv = np.linalg.svd(M.double().numpy(), compute_uv=False)
    big = np.sort(s)[::-1]
    # fp32 storage: the largest singular values match to fp32 accuracy
    assert np.allclose(sv[:16], big[:16], rtol=1e-5)
    # same seeds, same matrix; another matrix differs
    assert torch.equal(M, I.stress_momentum_torch(wl, idx, "cpu"))
    assert not torch.equal(M[:8, :8], I.stress_momentum_torch(wl, idx + 1, "cpu")[:8, :8])
