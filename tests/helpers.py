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
