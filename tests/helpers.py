"""Shared test utilities: tensor <-> float64 conversion, error metrics, input placement.

No arithmetic of the optimizer lives here; expected values always come from the
oracle package.
"""
from __future__ import annotations

import numpy as np
import torch

from muon_newton_schulz_07_b200 import inputs as I


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a (bf16 / fp32) tensor to float64 on the host."""
    return t.detach().to("cpu", torch.float64).numpy()


def rel_fro(a, b) -> float:
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a))


def bf16_ulp(x) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits), for |x| in the normal range."""
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 1e-37)))
    return np.exp2(e - 7)


def device_tensor(a: np.ndarray, dtype: torch.dtype, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device).to(dtype).contiguous()


def workload_tensors(wl: I.Workload, dtype, step=1, device="cuda", idx=None):
    """W, G, M of a workload (or of the listed matrix indices) as device tensors."""
    idx = range(len(wl.shapes)) if idx is None else idx
    W = [device_tensor(I.weight(wl, i), dtype, device) for i in idx]
    G = [device_tensor(I.gradient(wl, step, i), dtype, device) for i in idx]
    M = [device_tensor(I.momentum(wl, i), dtype, device) for i in idx]
    return W, G, M


def storage_ulp(x, dtype) -> np.ndarray:
    """Spacing of the storage type (bf16: 8 significant bits; fp32: 24) at |x|, normal range."""
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 1e-37)))
    return np.exp2(e - (7 if dtype == torch.bfloat16 else 23))


# The kernels evaluate each element in fp32 (a product and a fused multiply-add, with beta,
# 1 - beta and lr * s themselves rounded to fp32) before the one rounding to the storage type:
# a few units of 2^-24 of the summands' magnitudes, bounded here by 2^-21.
FP32_SLACK = 2.0 ** -21


def assert_m1_elementwise(M1_gpu, M1_ref, M0, G0, dtype, what="M1"):
    """Every element of M1 = beta M + (1 - beta) G, rounded once to the storage type, lies within
    half a storage spacing of the exact value (plus the fp32 arithmetic before that rounding)."""
    M1_gpu, M1_ref = np.asarray(M1_gpu, np.float64), np.asarray(M1_ref, np.float64)
    err = np.abs(M1_gpu - M1_ref)
    bound = 0.5 * storage_ulp(M1_ref, dtype) + FP32_SLACK * (np.abs(M0) + np.abs(G0))
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} elements off, worst excess " \
                          f"{float(np.max(err - bound)):.3e}"


def assert_w1_elementwise(W1_gpu, W1_ref, Wz_gpu, Wz_ref, W0, dtype, what="W1"):
    """W1 = round(d W + c O) with O the kernel's own direction as it applies it.  A step from the same
    momentum with W = 0 stores Wz = round(c O), so per element |c O - Wz_ref| <= |Wz - Wz_ref| +
    half a spacing of Wz, where Wz_ref is the oracle's step from W = 0.  W1 may then differ from
    the oracle's W1 by that direction error plus its own rounding (half a spacing)."""
    W1_gpu, W1_ref = np.asarray(W1_gpu, np.float64), np.asarray(W1_ref, np.float64)
    Wz_gpu, Wz_ref = np.asarray(Wz_gpu, np.float64), np.asarray(Wz_ref, np.float64)
    err = np.abs(W1_gpu - W1_ref)
    bound = (0.5 * storage_ulp(np.maximum(np.abs(W1_gpu), np.abs(W1_ref)), dtype) + np.abs(Wz_gpu - Wz_ref)
             + 0.5 * storage_ulp(Wz_gpu, dtype) + FP32_SLACK * (np.abs(W0) + np.abs(Wz_ref)))
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} elements off, worst excess " \
                          f"{float(np.max(err - bound)):.3e}"


def step_with_direction(op, W, G, M, **hp):
    """Run the step on (0, G, copy of M), then on (W, G, M).

    The first call writes round(-lr s O) into the zero matrices: the direction O the second call
    applies, since both start from the same momentum (the step is deterministic).  Returns those
    zero-start results; W and M are updated in place by the second call.
    """
    Wz = [torch.zeros_like(w) for w in W]
    Mz = [m.clone() for m in M]
    op(Wz, G, Mz, **hp)
    op(W, G, M, **hp)
    torch.cuda.synchronize()
    for a, b in zip(M, Mz):
        assert torch.equal(a, b), "two steps from the same momentum must give the same M1"
    return Wz
