"""GPU parity of the step's less common branches against the float64 oracle, element by element.

* nesterov = False (U = M1), and beta other than 0.95;
* weight decay != 0 on every parameter-write path: fused into the last Update (bf16 parameters
  whose dimensions are all multiples of 32; 256-wide tiles, and 512-wide tiles for long k loops)
  and param_write_kernel (fp32 parameters, and bf16 sets
  with a dimension that is not a multiple of 32).  lr * wd = 0.002 is the usual setting, but with
  bf16 parameters 0.002 |W| is below half a bf16 spacing of W, so a decay factor of 0.9 is checked
  as well: there a wrong factor cannot hide in the rounding;
* a matrix whose gradient and momentum are both zero, with eps = 0 and with the default eps: its
  direction is zero, so only the weight decay acts (the oracle's reading of 0 / 0).

Each case steps twice from the same momentum, once from W and once from W = 0 (which stores
round(-lr s O)).  M1 and W1 are held to per-element bounds (helpers.assert_m1_elementwise,
assert_w1_elementwise); O is held to the relative Frobenius budget of its mode (2e-2 for the bf16
tensor-core path, 1e-4 for the fp32 reference mode) plus the rounding of its storage.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from muon_newton_schulz_07_b200 import binding as B
from muon_newton_schulz_07_b200.optimizer import MuonStep

from helpers import (assert_m1_elementwise, assert_w1_elementwise, device_tensor, rel_fro, step_with_direction,
                     storage_ulp, to_f64)

pytestmark = pytest.mark.gpu

TOL_O = {"fast": 2e-2, "fp32_ref": 1e-4}

# (name, shapes, storage dtype, mode, which write path the handle must take)
SETS = [
    ("fused_d24_shapes", [(1536, 1536), (1536, 6144), (6144, 1536)], torch.bfloat16, "fast", "fused"),
    # long k loops (m = 2048): the writing Update runs 256 x 512 tiles, its parameter write
    # staged from registers after the accumulator is handed back (wide and tall parameters)
    ("fused_wide_write", [(2048, 2048), (4096, 2048), (2048, 4096)], torch.bfloat16, "fast", "fused"),
    ("write_kernel_ragged_bf16", [(200, 328), (328, 200), (512, 768)], torch.bfloat16, "fast", "kernel"),
    ("write_kernel_fp32", [(256, 512), (512, 256), (320, 320)], torch.float32, "fast", "kernel"),
    ("fp32_reference_mode", [(257, 129), (130, 130)], torch.float32, "fp32_ref", "kernel"),
]

HPARAMS = [
    dict(lr=0.02, beta=0.9, weight_decay=0.0, nesterov=False),
    dict(lr=0.02, beta=0.95, weight_decay=0.1, nesterov=True),
    dict(lr=0.05, beta=0.5, weight_decay=2.0, nesterov=False),   # decay factor 0.9
]


def inputs(shapes, dtype, seed):
    rng = np.random.default_rng(seed)
    W = [device_tensor(0.02 * rng.standard_normal(s), dtype) for s in shapes]
    G = [device_tensor(1e-3 * rng.standard_normal(s), dtype) for s in shapes]
    M = [device_tensor(1e-3 * rng.standard_normal(s), dtype) for s in shapes]
    return W, G, M


def expected_launches(op, path, k):
    """Launches of one step on the write path the case is meant to exercise (momentum/norm and
    the norms' finishing pass, the iterations, then the write kernel unless it is fused into the
    last Update)."""
    if op._mode == B.MUON_MODE_FP32_REF:
        return 2 + 3 * k * op.n_groups + 1
    if path == "small":
        return 2 + 1 + 1   # every iteration in one launch, then the write kernel
    # the default schedule runs every iteration in one launch when every shape group is at most
    # 768 wide, else one launch per stage
    single = all(-(-min(s) // 256) * 256 <= 768 for s in op.shapes)
    return 2 + (1 if single else 3 * k) + (0 if path == "fused" else 1)


def check_step(shapes, dtype, mode, path, hp, seed, k=5, eps=1e-7, zero=()):
    W, G, M = inputs(shapes, dtype, seed)
    for i in zero:
        G[i].zero_()
        M[i].zero_()
    pre = [(to_f64(w), to_f64(g), to_f64(m)) for w, g, m in zip(W, G, M)]
    op = MuonStep(shapes, dtype=dtype, mode=mode)
    assert op.launches_per_step(k) == expected_launches(op, path, k)
    Wz = step_with_direction(op, W, G, M, ns_steps=k, eps=eps, **hp)
    assert op.status() == B.MUON_OK
    ohp = O.Hyper(lr=hp["lr"], beta=hp["beta"], weight_decay=hp["weight_decay"], eps=eps,
                  nesterov=hp["nesterov"], ns_steps=k)
    errs = []
    for i, ((W0, G0, M0), s) in enumerate(zip(pre, shapes)):
        W1r, M1r, Or = O.muon_step(W0, G0, M0, ohp)
        Wzr = O.parameter_write(np.zeros_like(W0), Or, ohp.lr, ohp.weight_decay)
        W1g, M1g, Wzg = to_f64(W[i]), to_f64(M[i]), to_f64(Wz[i])
        assert np.isfinite(W1g).all() and np.isfinite(M1g).all(), s
        assert_m1_elementwise(M1g, M1r, M0, G0, dtype, what=f"M1 {s}")
        assert_w1_elementwise(W1g, W1r, Wzg, Wzr, W0, dtype, what=f"W1 {s}")
        if i in zero:
            assert not Wzg.any(), s     # zero direction: nothing but the decay
            errs.append((0.0, s))
            continue
        O_gpu = Wzg / (-ohp.lr * O.shape_scale(*s))
        err = rel_fro(O_gpu, Or)
        rounding = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -23
        assert err < TOL_O[mode] + rounding, (s, err)
        errs.append((err, s))
    op.close()
    return errs


@pytest.mark.parametrize("hp", HPARAMS, ids=["plain_beta0.9", "nesterov_wd0.1", "plain_beta0.5_decay0.9"])
@pytest.mark.parametrize("name,shapes,dtype,mode,path", SETS, ids=[s[0] for s in SETS])
def test_branches_elementwise(name, shapes, dtype, mode, path, hp):
    errs = check_step(shapes, dtype, mode, path, hp, seed=21)
    print(f"{name} {hp}: " + " ".join(f"{s[0]}x{s[1]}:{e:.2e}" for e, s in errs))


# (shapes, dtype, mode, path): the single-launch small-matrix path, the tensor-core path with the
# fused write, and the fp32 reference mode; matrix 0 has zero gradient and momentum.
ZERO_SETS = [
    ([(256, 256), (200, 96)], torch.bfloat16, "fast", "small"),
    ([(512, 512), (1024, 256)], torch.bfloat16, "fast", "fused"),
    ([(256, 384), (130, 130)], torch.float32, "fp32_ref", "kernel"),
]


@pytest.mark.parametrize("eps", [0.0, 1e-7])
@pytest.mark.parametrize("shapes,dtype,mode,path", ZERO_SETS, ids=["small_path", "fused_write", "fp32_ref"])
def test_zero_direction_only_decays(shapes, dtype, mode, path, eps):
    hp = dict(lr=0.05, beta=0.9, weight_decay=0.3, nesterov=True)
    check_step(shapes, dtype, mode, path, hp, seed=5, eps=eps, zero=(0,))
    # the zero matrix's norm is reported as exactly 0 and the other matrix is unaffected
    W, G, M = inputs(shapes, dtype, 5)
    G[0].zero_()
    M[0].zero_()
    W0 = to_f64(W[0])
    op = MuonStep(shapes, dtype=dtype, mode=mode)
    op(W, G, M, ns_steps=5, eps=eps, **hp)
    torch.cuda.synchronize()
    assert op.status() == B.MUON_OK
    assert float(op.norms()[0]) == 0.0
    decayed = (1.0 - hp["lr"] * hp["weight_decay"]) * W0
    err = np.abs(to_f64(W[0]) - decayed)
    assert np.all(err <= 0.5 * storage_ulp(decayed, dtype) + 2.0 ** -21 * np.abs(W0))
    op.close()


@pytest.mark.parametrize("shapes", [[(1536, 1536), (1536, 6144), (6144, 1536)],
                                    [(2048, 2048), (4096, 2048), (2048, 4096)]],
                         ids=["256_wide_tiles", "512_wide_tiles"])
def test_fused_write_equals_write_kernel(shapes):
    # Every write path computes W1 = (1 - lr wd) W - lr s X_k from the same bf16 X_k with the same
    # fused multiply-add, so the write fused into the last Update (16-byte aligned parameters) and
    # param_write_kernel (the same parameters one element off a 16-byte boundary) agree bit for bit.
    hp = dict(lr=0.05, beta=0.9, weight_decay=2.0, nesterov=True)
    W, G, M = inputs(shapes, torch.bfloat16, 91)
    Wk = []
    for w in W:
        base = torch.empty(w.numel() + 1, dtype=w.dtype, device=w.device)
        view = base[1:].view(w.shape)
        view.copy_(w)
        assert view.data_ptr() % 16 != 0
        Wk.append(view)
    Mk = [m.clone() for m in M]
    op = MuonStep(shapes, dtype=torch.bfloat16)
    op(W, G, M, ns_steps=5, **hp)
    op(Wk, G, Mk, ns_steps=5, **hp)
    torch.cuda.synchronize()
    assert op.status() == B.MUON_OK
    for a, b in zip(M, Mk):
        assert torch.equal(a, b)
    bad = [i for i, (a, b) in enumerate(zip(W, Wk)) if not torch.equal(a, b)]
    assert not bad, bad
    op.close()
