"""gdn_prefill_noalloc: the prefill entry point for callers that cannot
allocate device memory (for example an operator plug-in inside a framework
that owns all device memory and hands it only input and output tensors).  It
takes no workspace; its scratch is a fixed array inside the library.

Checked through the C ABI against gdn_prefill with a caller-owned workspace.
The array keeps the previous call's contents, so the calls run back to back
on different inputs (other seeds, shapes and dtypes, the larger case both
before and after a smaller one): a read of stale scratch would then give a
wrong result.  This file is collected last on purpose.
"""
import ctypes

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


def _case(name, lens, H_qk, H_v, dtype, seed):
    case = inputs.make_prefill(name, lens, H_qk, H_v, dtype=dtype, seed=seed, s0=True)
    c = to_cuda(case)
    o_ref, S_ref = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"],
                               cu_seqlens=c["cu_seqlens"])
    torch.cuda.synchronize()
    return dict(c=c, T=case.T, N=case.N, H_qk=H_qk, H_v=H_v, dtype=dtype,
                o_ref=o_ref.float().cpu().double().numpy(), S_ref=S_ref.cpu().double().numpy())


def _check_noalloc(x):
    io = gdn.GDN_F32 if x["dtype"] == torch.float32 else gdn.GDN_BF16
    o = torch.full((x["T"], x["H_v"], 128), float("nan"), dtype=x["dtype"], device="cuda")
    S = torch.full((x["N"], x["H_v"], 128, 128), float("nan"), dtype=torch.float32,
                   device="cuda")
    st = _call_noalloc(x["c"], x["T"], x["H_qk"], x["H_v"], io, o, S)
    assert st == gdn.GDN_OK, gdn.status_string(st)
    torch.cuda.synchronize()
    assert o_err(o, x["o_ref"]) <= O_TOL
    assert s_err(S, x["S_ref"]) <= S_TOL


def test_noalloc_matches_workspace_entry_point_on_calls_in_a_row():
    big = _case("noalloc-big", [150, 77, 33], 2, 6, torch.float32, 77)
    small = _case("noalloc-small", [200], 1, 3, torch.bfloat16, 78)
    for x in (big, small, big, small):
        _check_noalloc(x)
    assert gdn.last_device_error() == gdn.GDN_OK


def test_noalloc_runs_unsplit_when_the_split_needs_more_than_the_array():
    cap = gdn.lib().gdn_prefill_noalloc_max_scratch_bytes()
    T, H_qk, H_v = 8192, 2, 6
    assert gdn.workspace_size(1, T, H_qk, H_v, 128, gdn.GDN_BF16) > cap
    assert gdn.lib().gdn_prefill_segmented_workspace_size(1, T, H_qk, H_v, 128, 128,
                                                         gdn.GDN_BF16, 1) <= cap
    x = _case("noalloc-unsplit", [T], H_qk, H_v, torch.bfloat16, 79)
    _check_noalloc(x)
    assert gdn.last_device_error() == gdn.GDN_OK


def test_noalloc_rejects_scratch_beyond_its_maximum():
    cap = gdn.lib().gdn_prefill_noalloc_max_scratch_bytes()
    H_qk, H_v = 16, 48
    per_token = (2 * H_qk + H_v) * 128 * 2
    T = cap // per_token + 64  # needs more scratch than the array holds, even unsplit
    assert gdn.lib().gdn_prefill_segmented_workspace_size(1, T, H_qk, H_v, 128, 128,
                                                         gdn.GDN_F32, 1) > cap
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    cu = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    c = dict(q=dummy, k=dummy, v=dummy, log_alpha=dummy, beta=dummy, S0=None, cu_seqlens=cu)
    st = _call_noalloc(c, T, H_qk, H_v, gdn.GDN_F32, dummy, None)
    assert st == gdn.GDN_ERR_WORKSPACE
