"""The workspace-free momentum/norm entry point against the workspace one.

muon_momentum_norm_static serves callers that cannot give the library device
memory (an allocator that must own every allocation, a fixed pool, code that may
not call cudaMalloc): its reduction scratch is a fixed array inside libmuon.so.
It must produce what muon_step's first stage produces: the same M1 and U, bit for
bit (same arithmetic, same rounding), and the same ||U||_F up to the order of the
fp32 summation.  Checked on two calls in a row, through the C ABI, with and without
the Nesterov blend; both calls are also checked against the float64 oracle (M1 and
U element by element within half a storage spacing, the norm to 1e-5).

This file is collected last on purpose (its name sorts last).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from muon_newton_schulz_07_b200 import binding as B
from muon_newton_schulz_07_b200.optimizer import MuonStep

from helpers import assert_m1_elementwise, to_f64

pytestmark = pytest.mark.gpu

NORM_RTOL = 1e-5  # fp32 sums of up to 2^28 squares in two different orders


def x0_of(op, shape, dtype):
    """U as muon_step left it in the workspace (oriented min x max, so transpose tall shapes back)."""
    g, slot = B.muon_get_matrix_slot(op.handle, 0)
    mp, np_, _, x0, _, _, _ = B.muon_get_group_buffers(op.handle, g)
    esz = 2 if dtype == torch.bfloat16 else 4
    off = x0 - op._ws.data_ptr() + slot * mp * np_ * esz
    X = op._ws[off:off + mp * np_ * esz].view(dtype).view(mp, np_)
    r, c = shape
    return X[:r, :c] if r <= c else X[:c, :r].t()


@pytest.mark.parametrize("nesterov", [True, False])
@pytest.mark.parametrize("shape,dtype,mode", [
    ((768, 3072), torch.bfloat16, "fast"),
    ((6144, 1536), torch.bfloat16, "fast"),
    ((200, 328), torch.bfloat16, "fast"),
    ((257, 129), torch.float32, "fp32_ref"),
    ((1, 5), torch.bfloat16, "fast"),
])
def test_static_matches_workspace_entry_point(shape, dtype, mode, nesterov):
    torch.manual_seed(0)
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream()
    W = torch.randn(shape, device=dev).mul_(0.02).to(dtype)
    M_ws = torch.randn(shape, device=dev).mul_(1e-3).to(dtype)
    M_st = M_ws.clone()
    U_st = torch.empty(shape, device=dev, dtype=dtype)
    norm_st = torch.zeros(1, device=dev, dtype=torch.float32)
    op = MuonStep([shape], dtype=dtype, mode=mode)
    dt = B.MUON_BF16 if dtype == torch.bfloat16 else B.MUON_FP32
    for call in range(2):
        G = torch.randn(shape, device=dev).mul_(1e-3 * (call + 1)).to(dtype)
        G0, M0 = to_f64(G), to_f64(M_st)
        op([W], [G], [M_ws], lr=0.02, beta=0.95, nesterov=nesterov, ns_steps=1)
        B.muon_momentum_norm_static(G.data_ptr(), M_st.data_ptr(), U_st.data_ptr(), shape[0], shape[1], dt, 0.95,
                                    nesterov, norm_st.data_ptr(), stream.cuda_stream)
        torch.cuda.synchronize()
        assert op.status() == B.MUON_OK
        assert torch.equal(M_st, M_ws), call
        assert torch.equal(U_st, x0_of(op, shape, dtype)), call
        ref = float(op.norms()[0])
        got = float(norm_st[0])
        assert abs(got - ref) <= NORM_RTOL * ref, (call, got, ref)
        # and against the float64 oracle
        M1r = O.momentum_lerp(M0, G0, 0.95)
        Ur = O.nesterov_blend(G0, M1r, 0.95, nesterov)
        assert_m1_elementwise(to_f64(M_st), M1r, M0, G0, dtype, what=f"M1 call {call}")
        assert_m1_elementwise(to_f64(U_st), Ur, M0, G0, dtype, what=f"U call {call}")
        nr = O.frobenius_norm(Ur)
        assert abs(got - nr) <= NORM_RTOL * nr, (call, got, nr)
    op.close()


def test_static_rejects_sizes_beyond_its_scratch():
    n = int(np.sqrt(2.0 ** 29))
    with pytest.raises(B.MuonError) as e:
        B.muon_momentum_norm_static(16, 16, 16, n, n, B.MUON_BF16, 0.95, True, 16, 0)
    assert e.value.code == B.MUON_ERR_UNSUPPORTED
