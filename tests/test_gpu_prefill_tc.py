"""GPU parity of gdn_prefill_tc -- the prefill with its output state pass on
the fifth-generation tensor cores at every slice width -- and of
gdn_prefill_mma (the same pass on mma.sync, which gdn_prefill does not pick at
48-column slices) against the fp64 oracle, through the C ABI.  The cases reach all three slice widths of the pass (32, 48 and 64
columns: the width follows the number of (sequence, value head) units),
ragged and empty sequences, partial chunks, fp32 I/O, long-memory gates and
the segmented prefill, whose last phase also runs this pass."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_12_b200 import gdn, inputs
from tests.gpu_util import O_TOL, S_TOL, o_err, s_err, to_cuda

pytestmark = pytest.mark.gpu


def _tc(case):
    c = to_cuda(case)
    o, S = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"],
                       cu_seqlens=c["cu_seqlens"], state_pass="tcgen05")
    torch.cuda.synchronize()
    assert gdn.last_device_error() == gdn.GDN_OK
    return o, S


def _check(case, heads=None):
    o, S = _tc(case)
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, S0=case.S0,
                                  cu_seqlens=case.cu_seqlens, heads=heads)
    if heads is None:
        assert o_err(o, o_ref) <= O_TOL
        assert s_err(S, S_ref) <= S_TOL
    else:
        assert o_err(o[:, heads], o_ref[:, heads]) <= O_TOL
        assert s_err(S[:, heads], S_ref[:, heads]) <= S_TOL


@pytest.mark.parametrize("lens,H_qk,H_v,s0", [
    ([100, 0, 37, 64, 200], 2, 6, True),     # 30 units: 32-column slices
    ([1, 65, 128, 130], 1, 3, False),        # 12 units
    ([300] * 8, 2, 6, True),                 # 48 units: 48-column slices
    ([90] * 10, 2, 6, True),                 # 60 units: 64-column slices
])
def test_tc_prefill_matches_the_oracle(lens, H_qk, H_v, s0):
    _check(inputs.make_prefill("tc", lens, H_qk, H_v, seed=len(lens) * 7 + H_v, s0=s0))


def test_tc_prefill_fp32_io():
    case = inputs.make_prefill("tc_f32", [77, 150], 2, 4, dtype=torch.float32, seed=5, s0=True)
    o, _ = _tc(case)
    assert o.dtype == torch.float32
    _check(case)


def test_tc_prefill_long_memory():
    # alpha ~ 0.9975 per token: the state carries across all 24 chunks
    _check(inputs.make_prefill("tc_long", [1500], 2, 6, seed=9, s0=True, alpha_mu=-6.0))


def test_tc_prefill_benchmark_heads_4k_sampled():
    # 16/48 heads as in the benchmark layout, 4,096 tokens; sampled value heads
    _check(inputs.make_prefill("tc_4k", [4096], 16, 48, seed=3, s0=True), heads=[0, 17, 47])


def test_tc_prefill_segmented_long_few_heads():
    # one query/key head, three value heads, 8K tokens: the automatic choice splits
    # the sequence, and the last phase (from the pieces' entering states) is this pass
    case = inputs.make_prefill("tc_seg", [8192], 1, 3, seed=4, s0=True, alpha_mu=-6.0)
    assert gdn.auto_segments(1, 8192, 1, 3) > 1
    _check(case)


def test_tc_equals_default_within_rounding():
    case = inputs.make_prefill("tc_ab", [700, 333], 2, 6, seed=12, s0=True, alpha_mu=-3.0)
    c = to_cuda(case)
    o0, S0 = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"],
                         cu_seqlens=c["cu_seqlens"])
    o1, S1 = _tc(case)
    assert o_err(o1, o0.float().cpu().double().numpy()) <= O_TOL
    assert s_err(S1, S0.cpu().double().numpy()) <= S_TOL


@pytest.mark.parametrize("lens,H_qk,H_v", [([300] * 8, 2, 6), ([4096], 16, 48)])
def test_mma_pass_at_48_column_slices(lens, H_qk, H_v):
    # 48 units: gdn_prefill takes the tcgen05 pass here; the mma.sync one stays checked
    case = inputs.make_prefill("mma48", lens, H_qk, H_v, seed=17, s0=True)
    c = to_cuda(case)
    o, S = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"],
                       cu_seqlens=c["cu_seqlens"], state_pass="mma_sync")
    torch.cuda.synchronize()
    assert gdn.last_device_error() == gdn.GDN_OK
    heads = None if H_v <= 6 else [0, 25, 47]
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, S0=case.S0,
                                  cu_seqlens=case.cu_seqlens, heads=heads)
    if heads is None:
        assert o_err(o, o_ref) <= O_TOL and s_err(S, S_ref) <= S_TOL
    else:
        assert o_err(o[:, heads], o_ref[:, heads]) <= O_TOL
        assert s_err(S[:, heads], S_ref[:, heads]) <= S_TOL
