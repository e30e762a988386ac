"""The C ABI on a host without a GPU: the library builds, loads, exports every declared
symbol, sizes workspaces, and rejects bad arguments before touching a device."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from muon_newton_schulz_07_b200 import binding as B
from muon_newton_schulz_07_b200 import build as build_mod
from muon_newton_schulz_07_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    build_mod.build()
    return B.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "muon.h")).read()
    return sorted(set(re.findall(r"^MUON_API\s+[\w\s\*]*?\b(muon_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(B.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name


def test_status_strings():
    for code, name in B.STATUS.items():
        assert B.muon_status_string(code) == name
    assert B.muon_status_string(99) == "MUON_ERR_UNKNOWN"


def test_workspace_size_layout():
    # one group per orientation-free shape; X0, X1 (m x n) and A, B (m x m), padded to 256
    n1 = B.muon_workspace_size([(256, 256)], B.MUON_BF16, B.MUON_MODE_FAST)
    assert n1 >= 2 * 256 * 256 * 2 * 2
    tall_wide = B.muon_workspace_size([(512, 256), (256, 512)], B.MUON_BF16, B.MUON_MODE_FAST)
    wide = B.muon_workspace_size([(256, 512)], B.MUON_BF16, B.MUON_MODE_FAST)
    assert tall_wide - wide >= 2 * (2 * 256 * 512 + 2 * 256 * 256) - 4096
    ref = B.muon_workspace_size([(256, 256)], B.MUON_FP32, B.MUON_MODE_FP32_REF)
    assert ref > n1
    ragged = B.muon_workspace_size([(200, 328)], B.MUON_BF16, B.MUON_MODE_FAST)
    assert ragged >= 2 * 2 * 256 * 512 + 2 * 2 * 256 * 256


def test_workspace_size_d24():
    wl = I.WORKLOADS["d24"]
    n = B.muon_workspace_size(list(wl.shapes), B.MUON_BF16, B.MUON_MODE_FAST)
    x = I.param_count(wl) * 2 * 2
    a = 144 * 1536 * 1536 * 2 * 2
    assert x + a <= n <= x + a + 64 * 1024 * 1024


@pytest.mark.parametrize("shapes", [[], [(0, 4)], [(4, -1)]])
def test_workspace_size_rejects(shapes):
    with pytest.raises(B.MuonError) as e:
        B.muon_workspace_size(shapes, B.MUON_BF16, B.MUON_MODE_FAST)
    assert e.value.code == B.MUON_ERR_INVALID_ARG


def test_bad_dtype_and_mode():
    with pytest.raises(B.MuonError):
        B.muon_workspace_size([(8, 8)], 7, B.MUON_MODE_FAST)
    with pytest.raises(B.MuonError):
        B.muon_workspace_size([(8, 8)], B.MUON_BF16, 9)


def test_null_handle_calls():
    hp = B.make_hparams()
    lib = B.lib()
    assert lib.muon_step(None, None, None, None, ctypes.byref(hp), None) == B.MUON_ERR_INVALID_ARG
    assert lib.muon_orthogonalize(None, None, None, ctypes.byref(hp), None) == B.MUON_ERR_INVALID_ARG
    assert lib.muon_get_status(None, None) == B.MUON_ERR_INVALID_ARG
    assert lib.muon_destroy(None) == B.MUON_ERR_INVALID_ARG
    assert lib.muon_get_norms(None, None, None) == B.MUON_ERR_INVALID_ARG


def test_create_without_device_or_workspace():
    import torch

    if torch.cuda.is_available():
        pytest.skip("host has a GPU")
    with pytest.raises(B.MuonError) as e:
        B.muon_create([(256, 256)], B.MUON_BF16, B.MUON_MODE_FAST, 1 << 20, 1 << 30)
    assert e.value.code in (B.MUON_ERR_NO_DEVICE, B.MUON_ERR_CUDA)


def test_adamw_arguments_checked_on_host():
    # validation happens before any device work, so this runs without a GPU
    ok = B.AdamWHParams(1e-3, 0.9, 0.95, 1e-8, 0.0, 1)
    B.muon_adamw_step([], [], [], [], [], B.MUON_BF16, ok, 0)  # empty: no-op
    lib = B.lib()
    bad = B.AdamWHParams(1e-3, 0.9, 0.95, 1e-8, 0.0, 0)  # step counts from 1
    with pytest.raises(B.MuonError) as e:
        B.muon_adamw_step([16], [16], [16], [16], [8], B.MUON_BF16, bad, 0)
    assert e.value.code == B.MUON_ERR_INVALID_ARG
    with pytest.raises(B.MuonError):
        B.muon_adamw_step([16], [16], [16], [16], [-1], B.MUON_BF16, ok, 0)
    assert lib is not None


@pytest.mark.parametrize("num_sms", [148, 132, 8])
@pytest.mark.parametrize("k", [1, 2, 5, 10])
@pytest.mark.parametrize("name", ["d24", "gpt2s", "l38b", "stress", "single256"])
def test_launch_tables_are_consistent(name, k, num_sms):
    # the host-built tables of the persistent momentum/norm kernel and of the single-launch
    # Newton-Schulz schedule, checked by the library itself (no device needed)
    shapes = list(I.WORKLOADS[name].shapes)
    assert B.muon_check_plan(shapes, k, num_sms) == 0


@pytest.mark.parametrize("shapes", [
    [(200, 328), (328, 200), (520, 1000), (300, 300)],
    [(256, 512), (512, 768), (768, 1024), (1024, 256), (300, 1300), (512, 512)],
    [(8, 8), (1, 300), (300, 1), (130, 130)],
    [(1536, 1536)] * 200 + [(256, 4096)] * 3,
])
def test_launch_tables_ragged_and_many(shapes):
    for k in (1, 3, 5):
        assert B.muon_check_plan(shapes, k, 148) == 0
