"""GPU parity of the segmented prefill (sequence parallelism within one GPU):
each sequence cut into pieces that run side by side, joined by an exact scan
of the pieces' affine state maps.  Checked against the fp64 oracle and
against the unsegmented prefill, through the C ABI.

With the default gates (log alpha = -softplus(N(0, 1)), alpha ~ 0.5) the state
is forgotten within a chunk, so the pieces barely depend on one another; the
cases that test the join use long-memory gates (alpha_mu = -6: alpha ~ 0.9975
per token, the state survives thousands of tokens)."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_12_b200 import gdn, inputs
from tests.gpu_util import O_TOL, S_TOL, o_err, s_err, to_cuda

pytestmark = pytest.mark.gpu


def _both(case, segments):
    c = to_cuda(case)
    o, S = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"],
                       cu_seqlens=c["cu_seqlens"], segments=segments)
    torch.cuda.synchronize()
    assert gdn.last_device_error() == gdn.GDN_OK
    return o, S


@pytest.mark.parametrize("segments", [2, 3, 5])
def test_segmented_varlen_with_state_matches_the_oracle(segments):
    # ragged lengths, an empty sequence, one shorter than a chunk, nonzero S0
    case = inputs.make_prefill("seg_varlen", [700, 0, 1000, 50, 1291], 2, 6, seed=51, s0=True,
                               alpha_mu=-6.0)
    o, S = _both(case, segments)
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, S0=case.S0,
                                  cu_seqlens=case.cu_seqlens)
    assert o_err(o, o_ref) <= O_TOL
    assert s_err(S, S_ref) <= S_TOL


def test_segmented_equals_unsegmented():
    case = inputs.make_prefill("seg_vs_plain", [2048, 1111], 1, 3, seed=52, s0=True,
                               alpha_mu=-6.0)
    o1, S1 = _both(case, 1)
    o4, S4 = _both(case, 4)
    assert (o4.float() - o1.float()).abs().max().item() <= 1e-2 * o1.float().abs().max().item()
    assert ((S4 - S1).norm() / S1.norm()).item() <= 1e-2


def test_more_segments_than_chunks_leaves_empty_pieces():
    # 3 chunks cut into 8 pieces: the trailing pieces are empty (identity maps)
    case = inputs.make_prefill("seg_empty", [150], 1, 2, seed=53, s0=True, alpha_mu=-6.0)
    o, S = _both(case, 8)
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, S0=case.S0,
                                  cu_seqlens=case.cu_seqlens)
    assert o_err(o, o_ref) <= O_TOL
    assert s_err(S, S_ref) <= S_TOL


def test_segmented_fp32_io():
    case = inputs.make_prefill("seg_f32", [900, 333], 1, 2, seed=54, s0=True,
                               dtype=torch.float32, alpha_mu=-6.0)
    o, S = _both(case, 3)
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, S0=case.S0,
                                  cu_seqlens=case.cu_seqlens)
    assert o_err(o, o_ref) <= O_TOL
    assert s_err(S, S_ref) <= S_TOL


def test_tensor_parallel_shard_32k_splits_automatically():
    # the heads of one GPU under 8-way tensor parallelism (2 QK / 6 V heads), L = 32K:
    # 24 blocks would leave most SMs idle, so the library splits the sequence
    L, H_qk, H_v = 32768, 2, 6
    assert gdn.auto_segments(1, L, H_qk, H_v) > 1
    case = inputs.make_prefill("tp8_shard_32k", [L], H_qk, H_v, seed=55)
    o, S = _both(case, None)
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta,
                                  cu_seqlens=case.cu_seqlens)
    assert o_err(o, o_ref) <= O_TOL
    assert s_err(S, S_ref) <= S_TOL


def test_long_memory_shard_splits_and_joins_exactly():
    # long memory: each piece's entering state carries the earlier pieces' writes
    L, H_qk, H_v = 16384, 2, 6
    assert gdn.auto_segments(1, L, H_qk, H_v) > 1
    case = inputs.make_prefill("tp8_shard_16k_long", [L], H_qk, H_v, seed=56, s0=True,
                               alpha_mu=-6.0)
    o, S = _both(case, None)
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, S0=case.S0,
                                  cu_seqlens=case.cu_seqlens)
    assert o_err(o, o_ref) <= O_TOL
    assert s_err(S, S_ref) <= S_TOL
    # the last piece's rows depend on the join: check them on their own too
    tail = np.zeros(L, dtype=bool)
    tail[-L // 8:] = True
    assert o_err(o, o_ref, tail) <= O_TOL


def test_wide_batches_are_not_split():
    assert gdn.auto_segments(1, 32768, 16, 48) == 1
    assert gdn.auto_segments(8, 8 * 4096, 16, 48) == 1
