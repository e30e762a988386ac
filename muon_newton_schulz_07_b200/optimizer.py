"""PyTorch-facing wrapper of libmuon: torch allocates the workspace and provides the stream.

    step = MuonStep([(1536, 1536), (1536, 6144), ...], dtype=torch.bfloat16)
    step(W_list, G_list, M_list, lr=0.02, beta=0.95)      # W and M updated in place

Only argument checking and pointer marshalling happen here; the optimizer step
itself runs in libmuon's kernels on the current CUDA stream.
"""
from __future__ import annotations

import torch

from . import binding as B

QUINTIC = (3.4445, -4.7750, 2.0315)


class MuonStep:
    """A Muon step for one fixed list of matrix shapes, bound to one CUDA device."""

    SCHEDULES = {"auto": B.MUON_SCHEDULE_AUTO, "staged": B.MUON_SCHEDULE_STAGED, "fused": B.MUON_SCHEDULE_FUSED,
                 "split": B.MUON_SCHEDULE_SPLIT}

    def __init__(self, shapes, dtype=torch.bfloat16, mode: str = "fast", device=None, schedule: str = "auto"):
        if dtype not in (torch.bfloat16, torch.float32):
            raise TypeError("dtype must be torch.bfloat16 or torch.float32")
        if mode not in ("fast", "fp32_ref"):
            raise ValueError("mode must be 'fast' or 'fp32_ref'")
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.dtype = dtype
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self._dt = B.MUON_BF16 if dtype == torch.bfloat16 else B.MUON_FP32
        self._mode = B.MUON_MODE_FAST if mode == "fast" else B.MUON_MODE_FP32_REF
        nbytes = B.muon_workspace_size(self.shapes, self._dt, self._mode)
        self.workspace_bytes = nbytes
        with torch.cuda.device(self.device):
            self._ws = torch.empty(nbytes + 1024, dtype=torch.uint8, device=self.device)
            base = self._ws.data_ptr()
            self._ws_ptr = (base + 1023) // 1024 * 1024
            self.handle = B.muon_create(self.shapes, self._dt, self._mode, self._ws_ptr, nbytes)
        self.n_groups, _ = B.muon_get_plan(self.handle, 5)
        if schedule != "auto":
            self.set_schedule(schedule)

    def set_schedule(self, schedule: str) -> None:
        """'auto', 'staged' (one launch per Newton-Schulz stage), 'fused' (every iteration in one launch)
        or 'split' (the fused kernel's tiles, one launch per stage)."""
        if schedule not in self.SCHEDULES:
            raise ValueError(f"schedule must be one of {sorted(self.SCHEDULES)}")
        B.muon_set_schedule(self.handle, self.SCHEDULES[schedule])

    def launches_per_step(self, ns_steps: int = 5) -> int:
        return B.muon_get_plan(self.handle, ns_steps)[1]

    def _check(self, tensors, name):
        if len(tensors) != len(self.shapes):
            raise ValueError(f"{name}: expected {len(self.shapes)} tensors, got {len(tensors)}")
        for t, s in zip(tensors, self.shapes):
            if tuple(t.shape) != s or t.dtype != self.dtype or t.device != self.device or not t.is_contiguous():
                raise ValueError(f"{name}: tensor {tuple(t.shape)} {t.dtype} {t.device} does not match {s} "
                                 f"{self.dtype} {self.device} (contiguous)")
        return [t.data_ptr() for t in tensors]

    def __call__(self, W, G, M, lr=0.02, beta=0.95, weight_decay=0.0, eps=1e-7, abc=QUINTIC, nesterov=True,
                 ns_steps=5, stream=None):
        hp = B.make_hparams(lr, beta, weight_decay, eps, abc, nesterov, ns_steps)
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        B.muon_step(self.handle, self._check(W, "W"), self._check(G, "G"), self._check(M, "M"), hp, s.cuda_stream)

    def step_from_host(self, W, G_host, M, stream=None, **hp):
        """A step whose gradients are in pinned host memory.

        The host-to-device copy of G runs on a side stream into one of two device buffers,
        so it overlaps the previous step's kernels; the step itself waits for its copy.  The
        buffer is reused two steps later, once the step that read it has finished.  Keyword
        arguments are those of __call__.
        """
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        if getattr(self, "_gbuf", None) is None:
            self._gbuf = [[torch.empty(sh, dtype=self.dtype, device=self.device) for sh in self.shapes]
                          for _ in range(2)]
            self._copy_stream = torch.cuda.Stream(self.device)
            self._buf_free = [None, None]
            self._nfed = 0
        if len(G_host) != len(self.shapes):
            raise ValueError(f"G_host: expected {len(self.shapes)} tensors, got {len(G_host)}")
        b = self._nfed & 1
        cs = self._copy_stream
        with torch.cuda.stream(cs):
            if self._buf_free[b] is not None:
                cs.wait_event(self._buf_free[b])
            for d, h in zip(self._gbuf[b], G_host):
                if tuple(h.shape) != tuple(d.shape) or h.dtype != d.dtype:
                    raise ValueError(f"G_host: tensor {tuple(h.shape)} {h.dtype} does not match {tuple(d.shape)} "
                                     f"{d.dtype}")
                d.copy_(h, non_blocking=True)
            copied = torch.cuda.Event()
            copied.record(cs)
        s.wait_event(copied)
        self(W, self._gbuf[b], M, stream=s, **hp)
        done = torch.cuda.Event()
        done.record(s)
        self._buf_free[b] = done
        self._nfed += 1

    def host_copy_stream(self):
        """The side stream step_from_host copies on (created by its first call)."""
        return getattr(self, "_copy_stream", None)

    def orthogonalize(self, X, O, eps=1e-7, abc=QUINTIC, ns_steps=5, stream=None):
        hp = B.make_hparams(0.0, 0.0, 0.0, eps, abc, False, ns_steps)
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        B.muon_orthogonalize(self.handle, self._check(X, "X"), self._check(O, "O"), hp, s.cuda_stream)

    def norms(self, out=None, stream=None) -> torch.Tensor:
        """||U_i||_F of the last step, fp32, enqueued as one copy into `out` (device or pinned host)."""
        if out is None:
            out = torch.empty(len(self.shapes), dtype=torch.float32, device=self.device)
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        B.muon_get_norms(self.handle, out.data_ptr(), s.cuda_stream)
        return out

    def status(self, stream=None) -> int:
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        return B.muon_get_status(self.handle, s.cuda_stream)

    def close(self):
        if getattr(self, "handle", None):
            B.muon_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def adamw_step(params, grads, exp_avg, exp_avg_sq, step, lr=1e-3, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.0,
               stream=None):
    """AdamW on a list of tensors (bf16 or fp32 parameters, fp32 moments), one fused launch per 256 tensors.

    Every tensor must be contiguous and on the same CUDA device; `step` counts from 1.
    """
    if not params:
        return
    dt = params[0].dtype
    if dt not in (torch.bfloat16, torch.float32):
        raise TypeError("parameters must be bf16 or fp32")
    for p, g, m, v in zip(params, grads, exp_avg, exp_avg_sq):
        if not (p.is_contiguous() and g.is_contiguous() and m.is_contiguous() and v.is_contiguous()):
            raise ValueError("tensors must be contiguous")
        if p.dtype != dt or g.dtype != dt or m.dtype != torch.float32 or v.dtype != torch.float32:
            raise ValueError("p, g share the parameter dtype; moments are fp32")
        if not (p.numel() == g.numel() == m.numel() == v.numel()):
            raise ValueError("p, g, m, v must have equal sizes")
    hp = B.AdamWHParams(float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay), int(step))
    s = stream if stream is not None else torch.cuda.current_stream(params[0].device)
    B.muon_adamw_step([p.data_ptr() for p in params], [g.data_ptr() for g in grads],
                      [m.data_ptr() for m in exp_avg], [v.data_ptr() for v in exp_avg_sq],
                      [p.numel() for p in params], B.MUON_BF16 if dt == torch.bfloat16 else B.MUON_FP32, hp,
                      s.cuda_stream)
