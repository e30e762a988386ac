"""The single-launch schedule (every Newton-Schulz iteration in one persistent launch), and its
tiles run one launch per stage (the split schedule), against the staged schedule and the float64
oracle.

Both schedules run the same tiles with the same arithmetic: every accumulator receives the same
k slices in the same order and every epilogue rounds the same fp32 values, so their results must
be equal bit for bit; the staged schedule is itself checked against the oracle elsewhere, and a
few cases here are checked against the oracle directly.  The shape sets cover one and several
shape groups, 256- and 512-wide Update tiles (every group's padded width a multiple of 512, or
not), ragged sizes whose padding sits inside tiles, tall and wide matrices, the fused parameter
write and the separate write kernel, and k = 1, 2, 5.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from muon_newton_schulz_07_b200 import binding as B
from muon_newton_schulz_07_b200 import inputs as I
from muon_newton_schulz_07_b200.optimizer import MuonStep

from helpers import (assert_m1_elementwise, assert_w1_elementwise, device_tensor, rel_fro, step_with_direction,
                     to_f64)

pytestmark = pytest.mark.gpu

SETS = {
    # GPT-2-small shapes: 768-wide groups, 256-wide Update tiles
    "gpt2s_like": [(768, 768), (768, 768), (768, 3072), (3072, 768), (768, 768)],
    # d24 shapes: 512-wide Update tiles in every iteration but the one that writes W
    "d24_like": [(1536, 1536), (1536, 6144), (6144, 1536)],
    # ragged: padding inside tiles, separate write kernel (dimensions not multiples of 32)
    "ragged": [(200, 328), (328, 200), (520, 1000), (300, 300)],
    # six groups, the most one launch takes
    "six_groups": [(256, 512), (512, 768), (768, 1024), (1024, 256), (300, 1300), (512, 512)],
    # long k loops (m = 2048): the staged schedule's last Update writes O from 512-wide tiles, the
    # single launch from 256-wide ones; both from the same bf16 X_k
    "long_k": [(2048, 2048), (4096, 2048), (2048, 4096)],
}


def run(shapes, X, k, schedule, dtype=torch.bfloat16):
    op = MuonStep(shapes, dtype=dtype, schedule=schedule)
    Os = [torch.empty_like(x) for x in X]
    op.orthogonalize(X, Os, ns_steps=k)
    torch.cuda.synchronize()
    assert op.status() == B.MUON_OK
    launches = op.launches_per_step(k)
    op.close()
    return Os, launches


@pytest.mark.parametrize("k", [1, 2, 5])
@pytest.mark.parametrize("name", list(SETS))
def test_fused_schedule_equals_staged_bitwise(name, k):
    shapes = SETS[name]
    rng = np.random.default_rng(71)
    X = [device_tensor(rng.standard_normal(s), torch.bfloat16) for s in shapes]
    Of, lf = run(shapes, X, k, "fused")
    Os, ls = run(shapes, X, k, "staged")
    Op, lp = run(shapes, X, k, "split")
    # one launch for all iterations instead of 3 k (one per stage)
    assert ls - lf == 3 * k - 1 and lp == ls, (lf, ls, lp)
    for s, a, b, c in zip(shapes, Of, Os, Op):
        assert torch.equal(a, b), (name, k, s)
        assert torch.equal(c, b), (name, k, s)
    if k == 5:
        for s, x, o in zip(shapes, X, Of):
            err = rel_fro(to_f64(o), O.newton_schulz(to_f64(x), k))
            assert err < 2e-2 + 2.0 ** -8, (s, err)


@pytest.mark.parametrize("name", ["gpt2s_like", "d24_like"])
def test_fused_schedule_step_against_oracle(name):
    # a whole step (momentum, single-launch iterations, fused parameter write) element by element
    shapes = SETS[name]
    rng = np.random.default_rng(72)
    W = [device_tensor(0.02 * rng.standard_normal(s), torch.bfloat16) for s in shapes]
    G = [device_tensor(1e-3 * rng.standard_normal(s), torch.bfloat16) for s in shapes]
    M = [device_tensor(1e-3 * rng.standard_normal(s), torch.bfloat16) for s in shapes]
    pre = [(to_f64(w), to_f64(g), to_f64(m)) for w, g, m in zip(W, G, M)]
    op = MuonStep(shapes, dtype=torch.bfloat16, schedule="fused")
    hp = dict(lr=0.02, beta=0.95, weight_decay=0.1, nesterov=True)
    Wz = step_with_direction(op, W, G, M, ns_steps=5, **hp)
    assert op.status() == B.MUON_OK
    ohp = O.Hyper(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7, nesterov=True, ns_steps=5)
    for i, ((W0, G0, M0), s) in enumerate(zip(pre, shapes)):
        W1r, M1r, Or = O.muon_step(W0, G0, M0, ohp)
        Wzr = O.parameter_write(np.zeros_like(W0), Or, 0.02, 0.1)
        assert_m1_elementwise(to_f64(M[i]), M1r, M0, G0, torch.bfloat16)
        assert_w1_elementwise(to_f64(W[i]), W1r, to_f64(Wz[i]), Wzr, W0, torch.bfloat16)
        assert rel_fro(to_f64(Wz[i]) / (-0.02 * O.shape_scale(*s)), Or) < 2e-2 + 2.0 ** -8, s
    op.close()


def _full_gpt2s_steps(schedule, steps=2):
    wl = I.WORKLOADS["gpt2s"]
    n = len(wl.shapes)
    W = [device_tensor(I.weight(wl, i), torch.bfloat16) for i in range(n)]
    M = [device_tensor(I.momentum(wl, i), torch.bfloat16) for i in range(n)]
    op = MuonStep(wl.shapes, dtype=torch.bfloat16, schedule=schedule)
    for s in range(1, steps + 1):
        G = [device_tensor(I.gradient(wl, s, i), torch.bfloat16) for i in range(n)]
        op(W, G, M, ns_steps=5)
    torch.cuda.synchronize()
    assert op.status() == B.MUON_OK
    norms = op.norms().cpu()
    op.close()
    return W, M, norms


@pytest.mark.parametrize("schedule", ["staged", "fused", "split"])
def test_full_gpt2s_set_is_deterministic(schedule):
    # the same two steps twice give the same bits (the norms' partial sums are added in a fixed
    # order, every product accumulates its k slices in a fixed order)
    W1, M1, n1 = _full_gpt2s_steps(schedule)
    W2, M2, n2 = _full_gpt2s_steps(schedule)
    assert torch.equal(n1, n2)
    for a, b in zip(M1, M2):
        assert torch.equal(a, b)
    bad = [i for i, (a, b) in enumerate(zip(W1, W2)) if not torch.equal(a, b)]
    assert not bad, (schedule, bad)


def test_fused_schedule_full_gpt2s_set_equals_staged():
    # the whole GPT-2-small set (72 matrices, two groups) through one launch per step, two steps
    wl = I.WORKLOADS["gpt2s"]
    n = len(wl.shapes)
    W = [device_tensor(I.weight(wl, i), torch.bfloat16) for i in range(n)]
    M = [device_tensor(I.momentum(wl, i), torch.bfloat16) for i in range(n)]
    Gs = [[device_tensor(I.gradient(wl, s, i), torch.bfloat16) for i in range(n)] for s in (1, 2)]
    Wa, Ma = [w.clone() for w in W], [m.clone() for m in M]
    fused = MuonStep(wl.shapes, dtype=torch.bfloat16, schedule="fused")
    staged = MuonStep(wl.shapes, dtype=torch.bfloat16, schedule="staged")
    for G in Gs:
        fused(W, G, M, ns_steps=5)
        staged(Wa, G, Ma, ns_steps=5)
    torch.cuda.synchronize()
    assert fused.status() == B.MUON_OK and staged.status() == B.MUON_OK
    assert torch.equal(fused.norms(), staged.norms())
    for a, b in zip(M, Ma):
        assert torch.equal(a, b)
    bad = [(i, float((a.float() - b.float()).abs().max())) for i, (a, b) in enumerate(zip(W, Wa))
           if not torch.equal(a, b)]
    assert not bad, bad


def test_schedule_setting_is_checked():
    op = MuonStep([(256, 512)], dtype=torch.bfloat16)
    with pytest.raises(B.MuonError) as e:
        B.muon_set_schedule(op.handle, 7)
    assert e.value.code == B.MUON_ERR_INVALID_ARG
    ref = MuonStep([(256, 512)], dtype=torch.float32, mode="fp32_ref")
    with pytest.raises(B.MuonError) as e:
        B.muon_set_schedule(ref.handle, B.MUON_SCHEDULE_FUSED)
    assert e.value.code == B.MUON_ERR_UNSUPPORTED
    op.close()
    ref.close()
