"""GPU parity: libmuon (through its C ABI) against the float64 oracle on the same seeded inputs.

Tolerances (relative Frobenius error, max over matrices):
  * orthogonalised direction O:  2e-2 for the bf16 tensor-core path, 1e-4 for the fp32
    reference mode (fp32 FMA on the CUDA cores);
  * momentum M1: one rounding of the stored type per element, so 2^-8 (bf16) / 2^-23 (fp32)
    bounds the relative error of every element and hence of the Frobenius norm;
  * parameters W1 in bf16 storage: per element the result is rounded once (half a bf16
    spacing) and carries lr*s times the error of O, so
    ||W1 - W1_ref||_F <= 0.5 ||ulp(W1_ref)||_F * 1.01 + lr * s * 2e-2 * ||O_ref||_F.
    In fp32 storage (W1 - W)/(-lr*s) is O itself and is checked at O's tolerance.
Element by element, M1 lies within half a storage spacing of the oracle's value, and W1 within
half a spacing plus the direction error of that element (a second step from W = 0 stores the
direction the step applied; see helpers.assert_w1_elementwise).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle as O
from muon_newton_schulz_07_b200 import binding as B
from muon_newton_schulz_07_b200 import inputs as I
from muon_newton_schulz_07_b200.optimizer import MuonStep

from helpers import (assert_m1_elementwise, assert_w1_elementwise, bf16_ulp, device_tensor, rel_fro,
                     step_with_direction, to_f64, workload_tensors)

pytestmark = pytest.mark.gpu

TOL_O = {"fast": 2e-2, "fp32_ref": 1e-4}


def oracle_hp(lr=0.02, beta=0.95, wd=0.0, eps=1e-7, nesterov=True, k=5, abc=O.QUINTIC):
    return O.Hyper(lr=lr, beta=beta, weight_decay=wd, eps=eps, nesterov=nesterov, ns_steps=k, abc=abc)


def run_orthogonalize(shapes, Xs, dtype, mode, k=5, abc=O.QUINTIC, eps=1e-7):
    op = MuonStep(shapes, dtype=dtype, mode=mode)
    Os = [torch.empty_like(x) for x in Xs]
    op.orthogonalize(Xs, Os, eps=eps, abc=abc, ns_steps=k)
    torch.cuda.synchronize()
    assert op.status() == B.MUON_OK
    op.close()
    return Os


# ---------------------------------------------------------------- single 256x256 fp32 matrix

@pytest.mark.parametrize("mode", ["fp32_ref", "fast"])
def test_single256_step(mode):
    wl = I.WORKLOADS["single256"]
    W, G, M = workload_tensors(wl, torch.float32)
    W0, G0, M0 = to_f64(W[0]), to_f64(G[0]), to_f64(M[0])
    op = MuonStep(wl.shapes, dtype=torch.float32, mode=mode)
    Wz = step_with_direction(op, W, G, M, lr=0.02, beta=0.95, weight_decay=0.0, ns_steps=5)
    assert op.status() == B.MUON_OK
    W1r, M1r, Or = O.muon_step(W0, G0, M0, oracle_hp())
    assert rel_fro(to_f64(M[0]), M1r) < 2.0 ** -23
    assert_m1_elementwise(to_f64(M[0]), M1r, M0, G0, torch.float32)
    Wzr = O.parameter_write(np.zeros_like(W0), Or, 0.02, 0.0)
    assert_w1_elementwise(to_f64(W[0]), W1r, to_f64(Wz[0]), Wzr, W0, torch.float32)
    O_gpu = (to_f64(W[0]) - W0) / (-0.02 * O.shape_scale(256, 256))
    err = rel_fro(O_gpu, Or)
    print(f"single256 {mode}: O rel err {err:.3e}")
    # W1 - W loses ~2^-24 |W| / (lr |O|) of relative accuracy to cancellation
    tol = TOL_O[mode] + (2.0 ** -24) * np.linalg.norm(W0) / (0.02 * np.linalg.norm(Or))
    assert err < tol
    norms = op.norms().cpu().numpy()
    U = O.nesterov_blend(G0, M1r, 0.95, True)
    assert abs(norms[0] - O.frobenius_norm(U)) / O.frobenius_norm(U) < 1e-5


@pytest.mark.parametrize("mode", ["fp32_ref", "fast"])
def test_single256_cubic_polar(mode):
    # The cubic iteration converges to the polar factor; its step count follows the
    # smallest normalised singular value (see the oracle's pins).
    X = np.random.default_rng(0).standard_normal((256, 256)).astype(np.float32)
    s = np.linalg.svd(X.astype(np.float64), compute_uv=False)
    k = math.ceil(math.log(0.5 / (s[-1] / math.sqrt(np.sum(s * s)))) / math.log(1.5)) + 8
    k = min(k, 64)
    Xt = device_tensor(X, torch.float32)
    (Og,) = run_orthogonalize([(256, 256)], [Xt], torch.float32, mode, k=k, abc=O.CUBIC)
    ref = O.newton_schulz(X.astype(np.float64), k, O.CUBIC, 1e-7)
    err = rel_fro(to_f64(Og), ref)
    err_polar = rel_fro(to_f64(Og), O.polar_factor(X.astype(np.float64)))
    print(f"cubic {mode} k={k}: vs oracle {err:.3e}, vs polar {err_polar:.3e}")
    assert err < TOL_O[mode]


# ---------------------------------------------------------------- orthogonaliser on assorted shapes

SHAPES = [(256, 256), (256, 256), (200, 328), (328, 200), (512, 768), (768, 512), (64, 1000), (1000, 64),
          (8, 8), (1, 300), (300, 1), (130, 130)]


def out_rounding(dtype):
    # storing O rounds every element once: relative error <= 2^-8 (bf16), 2^-24 (fp32)
    return 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -24


@pytest.mark.parametrize("mode,dtype", [("fast", torch.bfloat16), ("fast", torch.float32),
                                        ("fp32_ref", torch.float32), ("fp32_ref", torch.bfloat16)])
@pytest.mark.parametrize("k", [1, 2, 5])
def test_orthogonalize_shapes(mode, dtype, k):
    rng = np.random.default_rng(11)
    Xs_np = [rng.standard_normal(s).astype(np.float32) for s in SHAPES]
    Xs = [device_tensor(x, dtype) for x in Xs_np]
    Os = run_orthogonalize(SHAPES, Xs, dtype, mode, k=k)
    a, b, c = O.QUINTIC
    errs = []
    for s, x, o in zip(SHAPES, Xs, Os):
        X = to_f64(x)
        ref = O.newton_schulz(X, k, O.QUINTIC, 1e-7)
        err = rel_fro(to_f64(o), ref)
        if mode == "fast" and k == 1:
            # One bf16 iteration rounds U, A, B and X once each (relative 2^-9 apiece).  B's
            # rounding reaches X through a X + B X, where a + b s^2 + c s^4 can cancel: it is
            # amplified by |b s^2 + c s^4| / |a + b s^2 + c s^4| at the largest normalised s.
            smax = np.linalg.norm(X, 2) / np.linalg.norm(X)
            y = smax * smax
            amp = abs(b * y + c * y * y) / abs(a + b * y + c * y * y)
            tol = 2.0 ** -9 * (3.0 + amp) * 1.25
        else:
            tol = TOL_O[mode]
        tol += out_rounding(dtype)
        errs.append((err, s))
        assert err < tol, (s, err, tol)
    print(f"orthogonalize {mode} {dtype} k={k}: " + " ".join(f"{s[0]}x{s[1]}:{e:.2e}" for e, s in errs))


# Every group's padded width (max dimension rounded up to 256) is a multiple of 512, so the
# Update runs on 256 x 512 pair tiles; ragged real sizes leave zero padding inside those tiles.
WIDE_SHAPES = [(256, 512), (512, 256), (300, 1000), (1000, 300), (512, 1024), (96, 480), (768, 1536)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("k", [1, 2, 5])
def test_orthogonalize_wide_update_tiles(dtype, k):
    rng = np.random.default_rng(17)
    Xs = [device_tensor(rng.standard_normal(s).astype(np.float32), dtype) for s in WIDE_SHAPES]
    Os = run_orthogonalize(WIDE_SHAPES, Xs, dtype, "fast", k=k)
    a, b, c = O.QUINTIC
    for s, x, o in zip(WIDE_SHAPES, Xs, Os):
        X = to_f64(x)
        ref = O.newton_schulz(X, k, O.QUINTIC, 1e-7)
        if k == 1:
            smax = np.linalg.norm(X, 2) / np.linalg.norm(X)
            y = smax * smax
            amp = abs(b * y + c * y * y) / abs(a + b * y + c * y * y)
            tol = 2.0 ** -9 * (3.0 + amp) * 1.25
        else:
            tol = TOL_O["fast"]
        tol += out_rounding(dtype)
        assert rel_fro(to_f64(o), ref) < tol, s


def test_intermediates_symmetric_and_padded():
    # Gram and polynomial matrices of the last iteration, read back from the workspace
    # (upper 256 x 256 blocks stored, the rest their transposes): zero outside the real
    # m x m block, and equal to the products of the normalised input within bf16 rounding.
    shapes = [(200, 328), (328, 200), (130, 130)]
    rng = np.random.default_rng(13)
    Xs = [device_tensor(rng.standard_normal(s), torch.bfloat16) for s in shapes]
    op = MuonStep(shapes, dtype=torch.bfloat16)
    Os = [torch.empty_like(x) for x in Xs]
    op.orthogonalize(Xs, Os, ns_steps=1)
    torch.cuda.synchronize()
    a, b, c = O.QUINTIC
    for i, x in enumerate(Xs):
        g, slot = B.muon_get_matrix_slot(op.handle, i)
        mp, np_, cnt, x0, x1, pa, pb = B.muon_get_group_buffers(op.handle, g)
        m = min(shapes[i])
        def view(ptr, rows, cols):
            # the buffers live inside the workspace tensor this test's MuonStep allocated
            off = ptr - op._ws.data_ptr() + slot * rows * cols * 2
            return to_f64(op._ws[off:off + rows * cols * 2].view(torch.bfloat16).view(rows, cols))
        def symmetric_from_upper(S):
            # only the 256 x 256 blocks on or above the diagonal are stored; the ones below
            # are their transposes
            F = S.copy()
            for I in range(mp // 256):
                for J in range(I):
                    F[I * 256:(I + 1) * 256, J * 256:(J + 1) * 256] = S[J * 256:(J + 1) * 256, I * 256:(I + 1) * 256].T
            return F
        As, Bs = view(pa, mp, mp), view(pb, mp, mp)
        A, Bm = symmetric_from_upper(As), symmetric_from_upper(Bs)
        for I in range(mp // 256):  # diagonal blocks are computed in full: symmetric to bf16 rounding
            d = slice(I * 256, (I + 1) * 256)
            assert np.all(np.abs(A[d, d] - A[d, d].T) <= bf16_ulp(A[d, d]))
            assert np.all(np.abs(Bm[d, d] - Bm[d, d].T) <= bf16_ulp(Bm[d, d]))
        assert not A[m:, :].any() and not A[:, m:].any()
        assert not Bm[m:, :].any() and not Bm[:, m:].any()
        U = to_f64(x)
        Xn = O.frobenius_normalize(U.T if U.shape[0] > U.shape[1] else U, 1e-7)
        A_ref = Xn @ Xn.T
        # the polynomial matrix carries the a X term of the update: B' = a I + b A + c A A
        B_ref = a * np.eye(m) + b * A_ref + c * (A_ref @ A_ref)
        assert rel_fro(A[:m, :m], A_ref) < 2 * 2.0 ** -8
        assert rel_fro(Bm[:m, :m], B_ref) < 4 * 2.0 ** -8


def test_orthogonalize_zero_steps_is_normalisation():
    rng = np.random.default_rng(12)
    shapes = [(256, 512), (384, 128)]
    Xs = [device_tensor(rng.standard_normal(s), torch.float32) for s in shapes]
    Os = run_orthogonalize(shapes, Xs, torch.float32, "fp32_ref", k=0)
    for x, o in zip(Xs, Os):
        assert rel_fro(to_f64(o), O.frobenius_normalize(to_f64(x), 1e-7)) < 1e-6


# ---------------------------------------------------------------- GPT-2-small set, several steps

def test_gpt2s_steps_teacher_forced():
    wl = I.WORKLOADS["gpt2s"]
    W, G, M = workload_tensors(wl, torch.bfloat16, step=1)
    op = MuonStep(wl.shapes, dtype=torch.bfloat16, mode="fast")
    check = [0, 4, 5, 6, 10, 11, 40, 71]  # Q, up, down of early and late layers
    for step in range(1, 4):
        if step > 1:
            G = [device_tensor(I.gradient(wl, step, i), torch.bfloat16) for i in range(len(wl.shapes))]
        pre = {i: (to_f64(W[i]), to_f64(G[i]), to_f64(M[i])) for i in check}
        Wz = step_with_direction(op, W, G, M, lr=0.02, beta=0.95, ns_steps=5)
        assert op.status() == B.MUON_OK
        for i in check:
            W0, G0, M0 = pre[i]
            W1r, M1r, Or = O.muon_step(W0, G0, M0, oracle_hp())
            assert rel_fro(to_f64(M[i]), M1r) < 2.0 ** -8
            assert_m1_elementwise(to_f64(M[i]), M1r, M0, G0, torch.bfloat16, what=f"M1 step {step} matrix {i}")
            r, c = wl.shapes[i]
            bound = 0.5 * 1.01 * np.linalg.norm(bf16_ulp(W1r)) + 0.02 * O.shape_scale(r, c) * 2e-2 * np.linalg.norm(Or)
            assert np.linalg.norm(to_f64(W[i]) - W1r) <= bound, (step, i)
            Wzr = O.parameter_write(np.zeros_like(W0), Or, 0.02, 0.0)
            assert rel_fro(to_f64(Wz[i]), Wzr) < 2e-2 + 2.0 ** -8, (step, i)
            assert_w1_elementwise(to_f64(W[i]), W1r, to_f64(Wz[i]), Wzr, W0, torch.bfloat16,
                                  what=f"W1 step {step} matrix {i}")


def test_gpt2s_orthogonal_direction():
    # The same momentum direction U the step would orthogonalise, through the NS-only entry point.
    wl = I.WORKLOADS["gpt2s"]
    idx = list(range(6))
    _, G, M = workload_tensors(wl, torch.bfloat16, step=1, idx=idx)
    U = []
    for g, m in zip(G, M):
        M1 = O.momentum_lerp(to_f64(m), to_f64(g), 0.95)
        U.append(device_tensor(O.nesterov_blend(to_f64(g), M1, 0.95, True), torch.bfloat16))
    shapes = [wl.shapes[i] for i in idx]
    Os = run_orthogonalize(shapes, U, torch.bfloat16, "fast")
    for u, o in zip(U, Os):
        err = rel_fro(to_f64(o), O.newton_schulz(to_f64(u), 5))
        assert err < TOL_O["fast"], err


# ---------------------------------------------------------------- determinism, resume, failure detection

def test_gpt2s_free_running_drift():
    # Ten steps with no teacher forcing: the GPU state and the oracle's (float64 from the same bf16
    # start, the same bf16 gradients) drift apart only through the per-step roundings.  W is stored
    # in bf16 every step (2^-9 relative) and M carries a 0.95 memory of its own roundings, so ten
    # steps stay near 1e-2; the drift is printed and held to 5e-2 (a wrong formula gives O(1)).
    wl = I.WORKLOADS["gpt2s"]
    idx = [0, 4, 5, 6, 10, 11]
    shapes = [wl.shapes[i] for i in idx]
    W, G, M = workload_tensors(wl, torch.bfloat16, step=1, idx=idx)
    Wr, Mr = [to_f64(w) for w in W], [to_f64(m) for m in M]
    op = MuonStep(shapes, dtype=torch.bfloat16)
    hp = oracle_hp()
    steps = 10
    for step in range(1, steps + 1):
        if step > 1:
            G = [device_tensor(I.gradient(wl, step, i), torch.bfloat16) for i in idx]
        Gr = [to_f64(g) for g in G]
        op(W, G, M, lr=0.02, beta=0.95, ns_steps=5)
        for j in range(len(idx)):
            Wr[j], Mr[j], _ = O.muon_step(Wr[j], Gr[j], Mr[j], hp)
    torch.cuda.synchronize()
    assert op.status() == B.MUON_OK
    dw = max(rel_fro(to_f64(w), wr) for w, wr in zip(W, Wr))
    dm = max(rel_fro(to_f64(m), mr) for m, mr in zip(M, Mr))
    print(f"gpt2s free-running drift after {steps} steps: W {dw:.2e}, M {dm:.2e}")
    assert dw < 5e-2 and dm < 5e-2


def test_deterministic_and_resumable():
    wl = I.WORKLOADS["gpt2s"]
    idx = list(range(6))
    shapes = [wl.shapes[i] for i in idx]
    W, G, M = workload_tensors(wl, torch.bfloat16, step=1, idx=idx)
    op = MuonStep(shapes, dtype=torch.bfloat16)
    Wa, Ma = [w.clone() for w in W], [m.clone() for m in M]
    op(Wa, G, Ma)
    op(Wa, G, Ma)
    ckW, ckM = [w.clone() for w in Wa], [m.clone() for m in Ma]  # checkpoint after 2 steps
    op(Wa, G, Ma)
    Wb, Mb = [w.clone() for w in W], [m.clone() for m in M]
    for _ in range(3):
        op(Wb, G, Mb)
    op(ckW, G, ckM)  # resume from the checkpoint
    torch.cuda.synchronize()
    for x, y, z in zip(Wa, Wb, ckW):
        assert torch.equal(x, y) and torch.equal(x, z)
    for x, y, z in zip(Ma, Mb, ckM):
        assert torch.equal(x, y) and torch.equal(x, z)


def test_timeout_is_reported_not_hung():
    op = MuonStep([(256, 256)], dtype=torch.bfloat16)
    s = torch.cuda.current_stream()
    B.muon_selftest_timeout(op.handle, 2_000_000, s.cuda_stream)  # 2 ms
    assert op.status() == B.MUON_ERR_TIMEOUT
    assert op.status() == B.MUON_OK  # read clears it
    # the context is still usable
    x = device_tensor(np.eye(256), torch.bfloat16)
    o = torch.empty_like(x)
    op.orthogonalize([x], [o], ns_steps=3)
    torch.cuda.synchronize()
    assert op.status() == B.MUON_OK


def test_invalid_arguments_rejected_before_launch():
    op = MuonStep([(256, 256)], dtype=torch.bfloat16)
    hp = B.make_hparams(ns_steps=65)
    x = torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.MuonError) as e:
        B.muon_step(op.handle, [x.data_ptr()], [x.data_ptr()], [x.data_ptr()], hp, 0)
    assert e.value.code == B.MUON_ERR_INVALID_ARG
    hp = B.make_hparams(beta=1.5)
    with pytest.raises(B.MuonError):
        B.muon_step(op.handle, [x.data_ptr()], [x.data_ptr()], [x.data_ptr()], hp, 0)
    with pytest.raises(B.MuonError):
        B.muon_step(op.handle, [x.data_ptr()], [None], [x.data_ptr()], B.make_hparams(), 0)
