"""gdn_prefill_noalloc: the prefill entry point for callers that cannot
allocate device memory (for example an operator plug-in inside a framework
that owns all device memory and hands it only input and output tensors).  It
takes no workspace; its scratch is a fixed array inside the library.

Checked through the C ABI against gdn_prefill with a caller-owned workspace,
on two calls in a row (the array keeps the previous call's contents, which
must not leak into the next result).  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_attention_12_b200 import gdn, inputs
from tests.gpu_util import O_TOL, S_TOL, o_err, s_err, to_cuda

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_noalloc(c, T, H_qk, H_v, io, o, S):
    N = c["cu_seqlens"].numel() - 1
    return gdn.lib().gdn_prefill_noalloc(
        _p(c["q"]), _p(c["k"]), _p(c["v"]), _p(c["log_alpha"]), _p(c["beta"]), _p(c["S0"]),
        _p(c["cu_seqlens"]), N, T, H_qk, H_v, 128, 128, io, _p(o), _p(S),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype,lens", [(torch.float32, [150, 77, 33]),
                                        (torch.bfloat16, [200])])
def test_noalloc_matches_workspace_entry_point_twice(dtype, lens):
    H_qk, H_v = 2, 6
    io = gdn.GDN_F32 if dtype == torch.float32 else gdn.GDN_BF16
    case = inputs.make_prefill("noalloc", lens, H_qk, H_v, dtype=dtype, seed=77, s0=True)
    c = to_cuda(case)
    T, N = case.T, case.N
    o_ref, S_ref = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"],
                               cu_seqlens=c["cu_seqlens"])
    for _ in range(2):
        o = torch.full((T, H_v, 128), float("nan"), dtype=dtype, device="cuda")
        S = torch.full((N, H_v, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
        st = _call_noalloc(c, T, H_qk, H_v, io, o, S)
        assert st == gdn.GDN_OK, gdn.status_string(st)
        torch.cuda.synchronize()
        assert o_err(o, o_ref.float().cpu().double().numpy()) <= O_TOL
        assert s_err(S, S_ref.cpu().double().numpy()) <= S_TOL
    assert gdn.last_device_error() == gdn.GDN_OK


def test_noalloc_rejects_scratch_beyond_its_maximum():
    cap = gdn.lib().gdn_prefill_noalloc_max_scratch_bytes()
    H_qk, H_v = 16, 48
    per_token = (2 * H_qk + H_v) * 128 * 2
    T = cap // per_token + 64  # needs more scratch than the array holds
    assert gdn.workspace_size(1, T, H_qk, H_v, 128, gdn.GDN_F32) > cap
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    cu = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    c = dict(q=dummy, k=dummy, v=dummy, log_alpha=dummy, beta=dummy, S0=None, cu_seqlens=cu)
    st = _call_noalloc(c, T, H_qk, H_v, gdn.GDN_F32, dummy, None)
    assert st == gdn.GDN_ERR_WORKSPACE
