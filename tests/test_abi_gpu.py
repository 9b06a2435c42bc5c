"""Argument rejection with a live CUDA context, through the raw C-ABI: host
pointers (pageable and pinned) are refused on the host before any launch, with
the offending argument named, and the context stays usable afterwards."""
from __future__ import annotations

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

cp = pytest.importorskip("lse_pack_stable_b200")
S = cp.Strides3
L = cp._lib


def _fused_raw(o_ptr, m_ptr, s_ptr, out_ptr, ol_ptr, W=2, T=4, H=8, D=64):
    return L.cp_pack_permute_combine_fused(o_ptr, S(T * H * D, H * D, D), m_ptr, S(T * H, H, 1),
                                           s_ptr, S(T * H, H, 1), W, T, H, D, 0, 1, out_ptr, ol_ptr,
                                           torch.cuda.current_stream().cuda_stream)


def test_host_and_pinned_pointers_are_rejected():
    W, T, H, D = 2, 4, 8, 64
    o = torch.randn(W, T, H, D, device="cuda", dtype=torch.bfloat16)
    m = torch.randn(W, T, H, device="cuda")
    s = torch.rand(W, T, H, device="cuda") + 1
    out = torch.empty(W, T, H // W, D, device="cuda", dtype=torch.bfloat16)
    ol = torch.empty(W, T, H // W, device="cuda")
    pageable = np.zeros(W * T * H * D, dtype=np.uint16)
    pinned = torch.empty(W * T * H * D, dtype=torch.int16, pin_memory=True)
    for bad in (pageable.ctypes.data, pinned.data_ptr()):
        st = _fused_raw(bad, m.data_ptr(), s.data_ptr(), out.data_ptr(), ol.data_ptr())
        assert st == cp.CP_ERR_ARG and "o is not device memory" in cp.last_error()
        st = _fused_raw(o.data_ptr(), m.data_ptr(), s.data_ptr(), bad, ol.data_ptr())
        assert st == cp.CP_ERR_ARG and "out is not device memory" in cp.last_error()
    # the context is fine: a valid call goes through and matches the binding
    assert _fused_raw(o.data_ptr(), m.data_ptr(), s.data_ptr(), out.data_ptr(), ol.data_ptr()) == 0
    ref, ref_l = cp.cp_pack_permute_combine_fused(o, m, s)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(ol, ref_l)
