"""Failure detection on the device, without a fault.

Every wait in the library's kernels is bounded in time; when one runs out the
kernel records GDN_ERR_TIMEOUT in the device status word and returns
normally.  gdn_selftest_bounded_wait makes such a wait run out on purpose (a
barrier that nothing arrives at); these tests check that the status is
reported once, then cleared, and that the context keeps working afterwards.
"""
import time

import pytest
import torch

import oracle
from linear_attention_12_b200 import gdn, inputs
from tests.gpu_util import O_TOL, S_TOL, o_err, s_err, to_cuda

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_is_reported_and_cleared():
    torch.cuda.synchronize()
    assert gdn.last_device_error() == gdn.GDN_OK
    t0 = time.monotonic()
    gdn.selftest_bounded_wait()
    st = gdn.last_device_error()
    elapsed = time.monotonic() - t0
    assert st == gdn.GDN_ERR_TIMEOUT, gdn.status_string(st)
    assert 1.0 < elapsed < 60.0  # the wait's limit is about 2 s
    assert gdn.last_device_error() == gdn.GDN_OK  # read and cleared


def test_the_context_stays_usable_after_a_timeout():
    gdn.selftest_bounded_wait()
    assert gdn.last_device_error() == gdn.GDN_ERR_TIMEOUT
    case = inputs.make_prefill("after_timeout", [100, 37], 2, 6, seed=11, s0=True)
    c = to_cuda(case)
    o, S = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"],
                       cu_seqlens=c["cu_seqlens"])
    torch.cuda.synchronize()
    assert gdn.last_device_error() == gdn.GDN_OK
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, S0=case.S0,
                                  cu_seqlens=case.cu_seqlens)
    assert o_err(o, o_ref) <= O_TOL
    assert s_err(S, S_ref) <= S_TOL
