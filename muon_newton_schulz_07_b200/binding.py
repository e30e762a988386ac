"""ctypes binding of libmuon.so: the C ABI of include/muon.h, same names, marshalling only.

Every function takes plain integers for device pointers, handles and streams and
returns what the C call returns (raising MuonError on a non-OK status).  No
arithmetic of the optimizer happens here: every step runs in the CUDA kernels.
If libmuon.so has not been built, the first call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmuon.so")

MUON_BF16, MUON_FP32 = 0, 1
MUON_MODE_FAST, MUON_MODE_FP32_REF = 0, 1

STATUS = {
    0: "MUON_OK",
    1: "MUON_ERR_INVALID_ARG",
    2: "MUON_ERR_UNSUPPORTED",
    3: "MUON_ERR_CUDA",
    4: "MUON_ERR_WORKSPACE",
    5: "MUON_ERR_TIMEOUT",
    6: "MUON_ERR_DEVICE_STATUS",
    7: "MUON_ERR_NO_DEVICE",
}
MUON_OK, MUON_ERR_INVALID_ARG, MUON_ERR_UNSUPPORTED, MUON_ERR_CUDA = 0, 1, 2, 3
MUON_ERR_WORKSPACE, MUON_ERR_TIMEOUT, MUON_ERR_DEVICE_STATUS, MUON_ERR_NO_DEVICE = 4, 5, 6, 7

KERNEL_KINDS = ("momentum_norm", "gram", "poly", "update", "write", "sgemm_ref", "ns_small", "ns_fused")
MUON_SCHEDULE_AUTO, MUON_SCHEDULE_STAGED, MUON_SCHEDULE_FUSED, MUON_SCHEDULE_SPLIT = 0, 1, 2, 3


class MuonError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class HParams(ctypes.Structure):
    _fields_ = [
        ("lr", ctypes.c_float),
        ("beta", ctypes.c_float),
        ("weight_decay", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("a", ctypes.c_float),
        ("b", ctypes.c_float),
        ("c", ctypes.c_float),
        ("nesterov", ctypes.c_int32),
        ("ns_steps", ctypes.c_int32),
    ]


_lib = None
_VP = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)


def lib() -> ctypes.CDLL:
    """Load libmuon.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m muon_newton_schulz_07_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        st = ctypes.c_int
        L.muon_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.POINTER(ctypes.c_size_t)]
        L.muon_workspace_size.restype = st
        L.muon_create.argtypes = [ctypes.POINTER(_VP), ctypes.POINTER(Shape), ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int, _VP, ctypes.c_size_t]
        L.muon_create.restype = st
        L.muon_step.argtypes = [_VP, _PP, _PP, _PP, ctypes.POINTER(HParams), _VP]
        L.muon_step.restype = st
        L.muon_orthogonalize.argtypes = [_VP, _PP, _PP, ctypes.POINTER(HParams), _VP]
        L.muon_orthogonalize.restype = st
        L.muon_get_norms.argtypes = [_VP, _VP, _VP]
        L.muon_get_norms.restype = st
        L.muon_get_status.argtypes = [_VP, _VP]
        L.muon_get_status.restype = st
        L.muon_selftest_timeout.argtypes = [_VP, ctypes.c_uint64, _VP]
        L.muon_selftest_timeout.restype = st
        L.muon_destroy.argtypes = [_VP]
        L.muon_destroy.restype = st
        L.muon_status_string.argtypes = [ctypes.c_int]
        L.muon_status_string.restype = ctypes.c_char_p
        L.muon_get_plan.argtypes = [_VP, ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        L.muon_get_plan.restype = st
        L.muon_get_matrix_slot.argtypes = [_VP, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                           ctypes.POINTER(ctypes.c_int)]
        L.muon_get_matrix_slot.restype = st
        L.muon_get_group_buffers.argtypes = [_VP, ctypes.c_int] + [ctypes.POINTER(ctypes.c_int)] * 3 + [_PP] * 4
        L.muon_get_group_buffers.restype = st
        L.muon_profile_begin.argtypes = [_VP, ctypes.c_int]
        L.muon_profile_begin.restype = st
        L.muon_profile_end.argtypes = [_VP, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int),
                                       ctypes.c_int]
        L.muon_profile_end.restype = st
        L.muon_set_schedule.argtypes = [_VP, ctypes.c_int]
        L.muon_set_schedule.restype = st
        _lib = L
    return _lib


def _check(code: int, where: str) -> None:
    if code != MUON_OK:
        raise MuonError(code, where)


def _shapes(shapes):
    arr = (Shape * len(shapes))()
    for i, (r, c) in enumerate(shapes):
        arr[i].rows, arr[i].cols = int(r), int(c)
    return arr


def _ptrs(ptrs):
    arr = (ctypes.c_void_p * len(ptrs))()
    for i, p in enumerate(ptrs):
        arr[i] = int(p) if p is not None else None
    return arr


def make_hparams(lr=0.02, beta=0.95, weight_decay=0.0, eps=1e-7, abc=(3.4445, -4.7750, 2.0315), nesterov=True,
                 ns_steps=5) -> HParams:
    return HParams(float(lr), float(beta), float(weight_decay), float(eps), float(abc[0]), float(abc[1]),
                   float(abc[2]), 1 if nesterov else 0, int(ns_steps))


def muon_workspace_size(shapes, dtype: int, mode: int) -> int:
    out = ctypes.c_size_t(0)
    arr = _shapes(shapes)
    _check(lib().muon_workspace_size(arr, len(shapes), dtype, mode, ctypes.byref(out)), "muon_workspace_size")
    return out.value


def muon_create(shapes, dtype: int, mode: int, workspace: int, ws_bytes: int) -> int:
    h = ctypes.c_void_p(None)
    arr = _shapes(shapes)
    _check(lib().muon_create(ctypes.byref(h), arr, len(shapes), dtype, mode, ctypes.c_void_p(workspace), ws_bytes),
           "muon_create")
    return h.value


def muon_step(handle: int, W, G, M, hp: HParams, stream: int) -> None:
    _check(lib().muon_step(handle, _ptrs(W), _ptrs(G), _ptrs(M), ctypes.byref(hp), ctypes.c_void_p(stream)),
           "muon_step")


def muon_orthogonalize(handle: int, X, O, hp: HParams, stream: int) -> None:
    _check(lib().muon_orthogonalize(handle, _ptrs(X), _ptrs(O), ctypes.byref(hp), ctypes.c_void_p(stream)),
           "muon_orthogonalize")


def muon_get_norms(handle: int, dst: int, stream: int) -> None:
    _check(lib().muon_get_norms(handle, ctypes.c_void_p(dst), ctypes.c_void_p(stream)), "muon_get_norms")


def muon_get_status(handle: int, stream: int) -> int:
    """Returns the raw status code (does not raise: a device fault is data here)."""
    return lib().muon_get_status(handle, ctypes.c_void_p(stream))


def muon_selftest_timeout(handle: int, timeout_ns: int, stream: int) -> None:
    _check(lib().muon_selftest_timeout(handle, int(timeout_ns), ctypes.c_void_p(stream)), "muon_selftest_timeout")


def muon_destroy(handle: int) -> None:
    _check(lib().muon_destroy(handle), "muon_destroy")


def muon_status_string(code: int) -> str:
    return lib().muon_status_string(code).decode()


def muon_get_plan(handle: int, ns_steps: int):
    g, l = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().muon_get_plan(handle, ns_steps, ctypes.byref(g), ctypes.byref(l)), "muon_get_plan")
    return g.value, l.value


def muon_check_plan(shapes, ns_steps: int, num_sms: int) -> int:
    """Number of inconsistencies in the host-built launch tables (0 when sound); no device needed."""
    L = lib()
    f = L.muon_check_plan
    f.argtypes = [ctypes.POINTER(Shape), ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int64)]
    f.restype = ctypes.c_int
    out = ctypes.c_int64(0)
    _check(f(_shapes(shapes), len(shapes), int(ns_steps), int(num_sms), ctypes.byref(out)), "muon_check_plan")
    return out.value


def muon_set_schedule(handle: int, schedule: int) -> None:
    _check(lib().muon_set_schedule(handle, int(schedule)), "muon_set_schedule")


def muon_profile_begin(handle: int, max_steps: int) -> None:
    _check(lib().muon_profile_begin(handle, int(max_steps)), "muon_profile_begin")


def muon_profile_end(handle: int):
    """{kind: (total_ms, launches)} for the calls traced since muon_profile_begin."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int * n)()
    _check(lib().muon_profile_end(handle, ms, cnt, n), "muon_profile_end")
    return {k: (ms[i], cnt[i]) for i, k in enumerate(KERNEL_KINDS)}


def muon_get_matrix_slot(handle: int, i: int):
    g, s = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().muon_get_matrix_slot(handle, i, ctypes.byref(g), ctypes.byref(s)), "muon_get_matrix_slot")
    return g.value, s.value


def muon_get_group_buffers(handle: int, group: int):
    """(mp, np, count, x0, x1, a, b) of a shape group; the last four are device addresses."""
    mp, np_, cnt = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    ptrs = [ctypes.c_void_p(None) for _ in range(4)]
    _check(lib().muon_get_group_buffers(handle, group, ctypes.byref(mp), ctypes.byref(np_), ctypes.byref(cnt),
                                        *[ctypes.byref(p) for p in ptrs]), "muon_get_group_buffers")
    return (mp.value, np_.value, cnt.value) + tuple(p.value for p in ptrs)


def muon_momentum_norm_static(G: int, M: int, U: int, rows: int, cols: int, dtype: int, beta: float,
                              nesterov: bool, norm: int, stream: int) -> None:
    L = lib()
    f = L.muon_momentum_norm_static
    f.argtypes = [_VP, _VP, _VP, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_int32, _VP,
                  _VP]
    f.restype = ctypes.c_int
    _check(f(ctypes.c_void_p(G), ctypes.c_void_p(M), ctypes.c_void_p(U), int(rows), int(cols), dtype, float(beta),
             1 if nesterov else 0, ctypes.c_void_p(norm), ctypes.c_void_p(stream)), "muon_momentum_norm_static")


class AdamWHParams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float), ("step", ctypes.c_int32)]


def muon_adamw_step(P, G, M, V, numel, dtype: int, hp: AdamWHParams, stream: int) -> None:
    L = lib()
    f = L.muon_adamw_step
    f.argtypes = [_PP, _PP, _PP, _PP, ctypes.POINTER(ctypes.c_int64), ctypes.c_int, ctypes.c_int,
                  ctypes.POINTER(AdamWHParams), _VP]
    f.restype = ctypes.c_int
    n = len(numel)
    sizes = (ctypes.c_int64 * max(n, 1))(*[int(x) for x in numel])
    _check(f(_ptrs(P), _ptrs(G), _ptrs(M), _ptrs(V), sizes, n, dtype, ctypes.byref(hp), ctypes.c_void_p(stream)),
           "muon_adamw_step")
