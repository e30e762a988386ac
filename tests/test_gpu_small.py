"""Sets whose matrices all fit one 256 x 256 tile: every Newton-Schulz iteration in one kernel.

The path is taken when each shape group pads to 256 x 256 (max(rows, cols) <= 256) and there
are at most six groups.  Against the float64 oracle with the bf16 path's tolerances (derived
for one iteration, 2e-2 after several), plus one rounding of the stored O.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from muon_newton_schulz_07_b200 import binding as B
from muon_newton_schulz_07_b200.optimizer import MuonStep

from helpers import device_tensor, rel_fro, to_f64

pytestmark = pytest.mark.gpu

# six groups, all padded to 256 x 256; ragged real sizes, a vector, a tiny matrix
SMALL_SHAPES = [(256, 256), (256, 256), (200, 100), (100, 200), (8, 8), (1, 256), (256, 1), (130, 130),
                (64, 256)]


def tolerance(X, k, dtype):
    a, b, c = O.QUINTIC
    if k == 1:
        smax = np.linalg.norm(X, 2) / np.linalg.norm(X)
        y = smax * smax
        amp = abs(b * y + c * y * y) / abs(a + b * y + c * y * y)
        tol = 2.0 ** -9 * (3.0 + amp) * 1.25
    else:
        tol = 2e-2
    return tol + (2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -24)


def launches_and_kinds(op, run):
    B.muon_profile_begin(op.handle, 1)
    run()
    prof = B.muon_profile_end(op.handle)
    return {k: v[1] for k, v in prof.items() if v[1]}


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("k", [1, 2, 5])
def test_small_set_orthogonalize(dtype, k):
    rng = np.random.default_rng(21)
    Xs = [device_tensor(rng.standard_normal(s).astype(np.float32), dtype) for s in SMALL_SHAPES]
    Os = [torch.empty_like(x) for x in Xs]
    op = MuonStep(SMALL_SHAPES, dtype=dtype)
    kinds = launches_and_kinds(op, lambda: op.orthogonalize(Xs, Os, ns_steps=k))
    torch.cuda.synchronize()
    assert op.status() == B.MUON_OK
    assert kinds.get("ns_small") == 1 and "gram" not in kinds, kinds
    for s, x, o in zip(SMALL_SHAPES, Xs, Os):
        X = to_f64(x)
        ref = O.newton_schulz(X, k, O.QUINTIC, 1e-7)
        err = rel_fro(to_f64(o), ref)
        assert err < tolerance(X, k, dtype), (s, k, err)


def test_small_set_many_matrices_per_pair():
    # 150 matrices: each CTA pair (74 of them) takes two or three in turn
    shapes = [(128, 96)] * 150
    rng = np.random.default_rng(22)
    Xs = [device_tensor(rng.standard_normal(s).astype(np.float32), torch.bfloat16) for s in shapes]
    Os = [torch.empty_like(x) for x in Xs]
    op = MuonStep(shapes)
    op.orthogonalize(Xs, Os, ns_steps=3)
    torch.cuda.synchronize()
    assert op.status() == B.MUON_OK
    for i in (0, 1, 73, 74, 75, 147, 148, 149):
        X = to_f64(Xs[i])
        ref = O.newton_schulz(X, 3, O.QUINTIC, 1e-7)
        assert rel_fro(to_f64(Os[i]), ref) < tolerance(X, 3, torch.bfloat16), i


def test_small_set_step_matches_oracle():
    # W = 0 leaves W1 = -lr sqrt(max(1, r/c)) O: the orthogonalised direction of the step
    rng = np.random.default_rng(23)
    shapes = SMALL_SHAPES
    G = [device_tensor(rng.standard_normal(s) * 1e-3, torch.bfloat16) for s in shapes]
    M = [device_tensor(rng.standard_normal(s) * 1e-3, torch.bfloat16) for s in shapes]
    W = [torch.zeros(s, device="cuda", dtype=torch.bfloat16) for s in shapes]
    pre = [(to_f64(g), to_f64(m)) for g, m in zip(G, M)]
    op = MuonStep(shapes)
    op(W, G, M, lr=0.02, beta=0.95, ns_steps=5)
    torch.cuda.synchronize()
    assert op.status() == B.MUON_OK
    hp = O.Hyper(lr=0.02, beta=0.95, weight_decay=0.0, eps=1e-7, nesterov=True, ns_steps=5)
    for s, (g0, m0), w, m in zip(shapes, pre, W, M):
        W1r, M1r, Or = O.muon_step(np.zeros(s), g0, m0, hp)
        assert rel_fro(to_f64(m), M1r) < 2.0 ** -8, s
        O_gpu = to_f64(w) / (-0.02 * O.shape_scale(*s))
        assert rel_fro(O_gpu, Or) < 2e-2 + 2.0 ** -8, s


def test_larger_sets_keep_the_general_path():
    # a set that does not fit one 256 x 256 tile per matrix leaves the small-matrix kernel: one
    # launch per stage when staged, one launch for every iteration by default (its groups are at
    # most 768 wide)
    staged = MuonStep([(256, 256), (256, 512)], schedule="staged")
    X = [torch.randn(s, device="cuda").to(torch.bfloat16) for s in staged.shapes]
    Os = [torch.empty_like(x) for x in X]
    kinds = launches_and_kinds(staged, lambda: staged.orthogonalize(X, Os, ns_steps=2))
    assert "ns_small" not in kinds and kinds.get("gram") == 2, kinds
    auto = MuonStep([(256, 256), (256, 512)])
    Oa = [torch.empty_like(x) for x in X]
    kinds = launches_and_kinds(auto, lambda: auto.orthogonalize(X, Oa, ns_steps=2))
    assert "ns_small" not in kinds and "gram" not in kinds and kinds.get("ns_fused") == 1, kinds
    for a, b in zip(Oa, Os):
        assert torch.equal(a, b)
