"""AdamW (the non-matrix half of the hybrid optimizer) against the float64 oracle, through the C ABI.

Per element the kernel works in fp32 and stores p once in its dtype and m, v in fp32, so:
  m1, v1:  |gpu - ref| <= 8 * 2^-24 * (|m| + |g|), resp. (|v| + g^2): a few fp32 roundings of
           the two summands (which may cancel in m1) and of beta passed as an fp32 number
  p1:      |gpu - ref| <= ulp(|ref|) + 1e-5 lr  (one rounding of the stored p, and the update
           lr * mh / (sqrt(vh) + eps), of size <= ~lr, computed in fp32 to a few 1e-7)
Each step is teacher-forced: the oracle starts from the GPU's own state before the step.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from muon_newton_schulz_07_b200 import binding as B
from muon_newton_schulz_07_b200.optimizer import adamw_step

from helpers import bf16_ulp, to_f64

pytestmark = pytest.mark.gpu

SIZES = [1, 7, 8, 2047, 2048, 2049, 100003, 3 * 65536]


def ulp(x, dtype):
    x = np.abs(np.asarray(x, np.float64))
    if dtype == torch.bfloat16:
        return bf16_ulp(x)
    return np.exp2(np.floor(np.log2(np.maximum(x, 1e-37))) - 23)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("misaligned", [False, True])
def test_adamw_matches_oracle(dtype, misaligned):
    torch.manual_seed(3)
    dev = torch.device("cuda")
    off = 1 if misaligned else 0  # a view one element in: pointers no longer 16-byte aligned
    P, G, M, V = [], [], [], []
    for n in SIZES:
        P.append(torch.randn(n + off, device=dev).to(dtype)[off:])
        G.append(torch.zeros(n + off, device=dev).to(dtype)[off:])
        M.append(torch.zeros(n + off, device=dev)[off:])
        V.append(torch.zeros(n + off, device=dev)[off:])
    lr, b1, b2, eps, wd = 3e-3, 0.9, 0.95, 1e-8, 0.1
    for step in range(1, 4):
        for g in G:
            g.copy_((torch.randn(g.numel(), device=dev) * (0.1 * step)).to(dtype))
        pre = [(to_f64(p), to_f64(g), to_f64(m), to_f64(v)) for p, g, m, v in zip(P, G, M, V)]
        adamw_step(P, G, M, V, step, lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
        torch.cuda.synchronize()
        for (p0, g0, m0, v0), p, m, v in zip(pre, P, M, V):
            p1, m1, v1 = O.adamw_step(p0, g0, m0, v0, step, lr, b1, b2, eps, wd)
            u = 2.0 ** -24
            assert np.all(np.abs(to_f64(m) - m1) <= 8 * u * (np.abs(m0) + np.abs(g0)) + 1e-30)
            assert np.all(np.abs(to_f64(v) - v1) <= 8 * u * (np.abs(v0) + g0 * g0) + 1e-30)
            assert np.all(np.abs(to_f64(p) - p1) <= ulp(p1, dtype) + 1e-5 * lr), (step, p.numel())


def test_adamw_rejects_bad_arguments():
    x = torch.zeros(16, device="cuda")
    ok = B.AdamWHParams(1e-3, 0.9, 0.95, 1e-8, 0.0, 1)
    for bad in (B.AdamWHParams(1e-3, 0.9, 0.95, 1e-8, 0.0, 0), B.AdamWHParams(1e-3, 1.0, 0.95, 1e-8, 0.0, 1),
                B.AdamWHParams(1e-3, 0.9, 0.95, -1.0, 0.0, 1)):
        with pytest.raises(B.MuonError):
            B.muon_adamw_step([x.data_ptr()], [x.data_ptr()], [x.data_ptr()], [x.data_ptr()], [16], B.MUON_FP32, bad,
                              0)
    with pytest.raises(B.MuonError):
        B.muon_adamw_step([x.data_ptr()], [None], [x.data_ptr()], [x.data_ptr()], [16], B.MUON_FP32, ok, 0)
    B.muon_adamw_step([], [], [], [], [], B.MUON_FP32, ok, 0)  # empty list: a no-op
