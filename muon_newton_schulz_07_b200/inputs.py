"""Seeded synthetic inputs for the Muon step: shapes, distributions, seeds.

This module draws random numbers and nothing else: it holds none of the
optimizer's arithmetic, and both the CUDA path's tests/bench and the oracle's
checks take their inputs from it.  Every tensor is a pure function of
(workload id, step, matrix index, tensor id) through
``numpy.random.SeedSequence([wid, step, idx, tid])``, so any single matrix can
be regenerated on its own (the oracle checks sampled matrices of the large
sets this way).

Workloads (shapes from the architectures the pages describe: nanochat d24 is
24 layers of width 1536, magicnetworld, FLOPs section; little-lm 3.8B is 28
layers of width 3072 with 24 query / 8 KV heads of dim 128 and a relu^2 MLP,
aiproducthub, 事件详情 paragraph):

  single256  1 x 256x256 fp32; W, G, M ~ N(0, 1)
  gpt2s      12 layers x {Q,K,V,O 768x768, up 768x3072, down 3072x768} = 72;
             G ~ N(0, 1e-3^2) with 1 % of entries x100, M ~ N(0, 1e-3^2)
  d24        24 layers x {Q,K,V,O 1536x1536, up 1536x6144, down 6144x1536} = 144;
             G row i ~ N(0, s_i^2), s_i = 10^U(-4,-2); M = 0
  l38b       28 layers x {Q,O 3072x3072, K,V 3072x1024, up 3072x12288,
             down 12288x3072} = 168; G, M ~ N(0, 1e-3^2)
  stress     64 each of 4096x512, 512x4096, 2048x2048, 8192x1024 = 256;
             M = P diag(s) Q^T, P, Q orthonormal (QR of Gaussians), s log-uniform
             in [1e-6, 1]; G = M
W ~ N(0, 0.02^2) everywhere except single256.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

TID_W, TID_G, TID_M, TID_P, TID_Q, TID_S, TID_MASK, TID_ROWSTD = 0, 1, 2, 3, 4, 5, 6, 7


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int
    shapes: tuple          # ((rows, cols), ...) in parameter order
    dtype: str             # storage dtype of W, G, M: "f32" or "bf16"
    steps: int             # consecutive optimizer steps the workload describes
    description: str


def _layers(n, per_layer):
    return tuple(s for _ in range(n) for s in per_layer)


WORKLOADS = {
    "single256": Workload("single256", 1, ((256, 256),), "f32", 1,
                          "one 256x256 fp32 matrix, N(0,1) W/G/M, seed 0"),
    "gpt2s": Workload("gpt2s", 2, _layers(12, [(768, 768)] * 4 + [(768, 3072), (3072, 768)]), "bf16", 10,
                      "GPT-2-small-shaped set, 72 matrices, heavy-tailed grads"),
    "d24": Workload("d24", 3, _layers(24, [(1536, 1536)] * 4 + [(1536, 6144), (6144, 1536)]), "bf16", 20,
                    "nanochat d24-shaped set, 144 matrices, per-row log-uniform grad std"),
    "l38b": Workload("l38b", 4, _layers(28, [(3072, 3072), (3072, 1024), (3072, 1024), (3072, 3072),
                                             (3072, 12288), (12288, 3072)]), "bf16", 1,
                     "3.8B-shaped GQA set, 168 matrices"),
    "stress": Workload("stress", 5, tuple([(4096, 512)] * 64 + [(512, 4096)] * 64 + [(2048, 2048)] * 64
                                          + [(8192, 1024)] * 64), "bf16", 1,
                       "aspect-ratio / conditioning stress set, 256 matrices, singular values in [1e-6, 1]"),
}


def rng_for(wid: int, step: int, idx: int, tid: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([wid, step, idx, tid]))


def normal(wid, step, idx, tid, shape, std=1.0) -> np.ndarray:
    x = rng_for(wid, step, idx, tid).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _orthonormal_columns(g: np.random.Generator, n: int, k: int) -> np.ndarray:
    q, r = np.linalg.qr(g.standard_normal((n, k)))
    return q * np.sign(np.diag(r))


def stress_factors(wid, idx, rows, cols):
    """(P, s, Q) with P: rows x k, Q: cols x k orthonormal, s log-uniform in [1e-6, 1]."""
    k = min(rows, cols)
    P = _orthonormal_columns(rng_for(wid, 0, idx, TID_P), rows, k)
    Q = _orthonormal_columns(rng_for(wid, 0, idx, TID_Q), cols, k)
    s = np.exp(rng_for(wid, 0, idx, TID_S).uniform(np.log(1e-6), 0.0, k))
    return P, s, Q


def stress_momentum_torch(wl: Workload, idx: int, device):
    """The stress set's matrix idx made on `device` with torch (same recipe, another stream).

    M = P diag(s) Q^T with P, Q the orthonormal factors of torch.linalg.qr of Gaussian matrices
    drawn by torch's generator (seeded from the same (workload, matrix, tensor) seeds), columns'
    signs fixed by diag(R), and s log-uniform in [1e-6, 1] (NumPy, as in stress_factors).  The
    values differ from momentum() (another random stream and QR), the structure does not.  QR of
    the 256 matrices on the host takes minutes; on a GPU it takes seconds, so the full-size GPU
    runs (tests and benchmark legs) draw the stress set here.  Returns a float32 tensor.
    """
    import torch

    r, c = wl.shapes[idx]
    k = min(r, c)

    def factor(n, tid):
        seed = int(np.random.SeedSequence([wl.wid, 0, idx, tid]).generate_state(1)[0])
        gen = torch.Generator(device=device).manual_seed(seed)
        a = torch.randn((n, k), generator=gen, device=device, dtype=torch.float64)
        q, rr = torch.linalg.qr(a)
        return q * torch.sign(torch.diagonal(rr))

    P, Q = factor(r, TID_P), factor(c, TID_Q)
    sv = np.exp(rng_for(wl.wid, 0, idx, TID_S).uniform(np.log(1e-6), 0.0, k))
    s = torch.from_numpy(sv).to(device)
    return ((P * s) @ Q.T).to(torch.float32)


def weight(wl: Workload, idx: int) -> np.ndarray:
    r, c = wl.shapes[idx]
    if wl.name == "single256":
        return normal(wl.wid, 0, idx, TID_W, (r, c))
    return normal(wl.wid, 0, idx, TID_W, (r, c), 0.02)


def momentum(wl: Workload, idx: int) -> np.ndarray:
    r, c = wl.shapes[idx]
    if wl.name == "single256":
        return normal(wl.wid, 0, idx, TID_M, (r, c))
    if wl.name == "d24":
        return np.zeros((r, c), np.float32)
    if wl.name == "stress":
        P, s, Q = stress_factors(wl.wid, idx, r, c)
        return ((P * s) @ Q.T).astype(np.float32)
    return normal(wl.wid, 0, idx, TID_M, (r, c), 1e-3)


def gradient(wl: Workload, step: int, idx: int) -> np.ndarray:
    r, c = wl.shapes[idx]
    if wl.name == "single256":
        return normal(wl.wid, step, idx, TID_G, (r, c))
    if wl.name == "gpt2s":
        g = normal(wl.wid, step, idx, TID_G, (r, c), 1e-3)
        mask = rng_for(wl.wid, step, idx, TID_MASK).random((r, c)) < 0.01
        g[mask] *= np.float32(100.0)
        return g
    if wl.name == "d24":
        g = normal(wl.wid, step, idx, TID_G, (r, c))
        std = np.power(10.0, rng_for(wl.wid, step, idx, TID_ROWSTD).uniform(-4.0, -2.0, r)).astype(np.float32)
        g *= std[:, None]
        return g
    if wl.name == "stress":
        return momentum(wl, idx)
    return normal(wl.wid, step, idx, TID_G, (r, c), 1e-3)


# The parameters of the d24 model that AdamW updates.  The magicnetworld page (FLOPs section) gives
# 1,384,124,976 parameters in all, 679,481,856 in the transformer matrices and 50,331,648 in the
# lm_head (32768 x 1536); the other 654,311,472 are not itemized there and are modelled as 13
# embedding tables of 32768 x 1536 plus 48 scalars.
D24_ADAMW_SIZES = tuple([32768 * 1536] * 14 + [1] * 48)


def adamw_param(step: int, idx: int, tid: int, n: int) -> np.ndarray:
    """Synthetic AdamW tensors: parameters N(0, 0.02^2), gradients N(0, 1e-3^2)."""
    std = 0.02 if tid == TID_W else 1e-3
    return normal(100, step, idx, tid, (n,), std)


def param_count(wl: Workload) -> int:
    return sum(r * c for r, c in wl.shapes)
