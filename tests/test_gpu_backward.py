"""GPU parity of gdn_prefill_backward (bf16 and fp32 I/O), and of the
training pair gdn_prefill_train + gdn_prefill_backward_saved, against the fp64 backward oracle
(oracle/backward.py), through the C ABI: every gradient on ragged packed
sequences, many-chunk sequences, grouped heads and long-memory gates.

Bar: max|g - g_ref| / max|g_ref| <= 1e-2 for each gradient (the forward's
bar for the output, applied to every gradient)."""
import numpy as np
import pytest
import torch

from linear_attention_12_b200 import gdn, inputs
from oracle import backward

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _case(name, lens, H_qk, H_v, seed, s0=True, with_dsf=True, alpha_mu=0.0,
          dtype=torch.bfloat16):
    case = inputs.make_prefill(name, lens, H_qk, H_v, seed=seed, s0=s0, alpha_mu=alpha_mu,
                               dtype=dtype)
    gen = torch.Generator().manual_seed(seed + 1000)
    T, N = case.q.shape[0], len(lens)
    dO = torch.randn((T, H_v, 128), generator=gen).to(dtype)
    dSf = 0.1 * torch.randn((N, H_v, 128, 128), generator=gen) if with_dsf else None
    return case, dO, dSf


def _check(case, dO, dSf, dtype=torch.bfloat16):
    d = lambda x: None if x is None else x.cuda()
    got = gdn.prefill_backward(d(case.q), d(case.k), d(case.v), d(case.log_alpha), d(case.beta),
                               d(dO), S0=d(case.S0), dS_final=d(dSf),
                               cu_seqlens=d(case.cu_seqlens))
    torch.cuda.synchronize()
    assert gdn.last_device_error() == gdn.GDN_OK
    ref = backward.prefill_backward(case.q, case.k, case.v, case.log_alpha, case.beta,
                                    dO.float().numpy(),
                                    S0=None if case.S0 is None else case.S0.numpy(),
                                    dS_final=None if dSf is None else dSf.numpy(),
                                    cu_seqlens=case.cu_seqlens.numpy())
    assert got[0].dtype == got[1].dtype == got[2].dtype == dtype
    for name, a, b in zip(["dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"], got, ref):
        a = a.float().cpu().double().numpy()
        err = np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)
        assert err <= TOL, (name, err)


@pytest.mark.parametrize("lens,H_qk,H_v", [([100, 0, 37, 64], 2, 6), ([192], 1, 3),
                                           ([1024], 1, 3), ([1024], 1, 1), ([300, 65], 2, 4)])
def test_backward_matches_the_oracle(lens, H_qk, H_v):
    _check(*_case("bw", lens, H_qk, H_v, seed=len(lens) + H_v))


def test_backward_without_initial_state_or_state_gradient():
    _check(*_case("bw_plain", [640], 1, 3, seed=7, s0=False, with_dsf=False))


def test_backward_long_memory():
    # alpha ~ 0.9975 per token: the state gradient carries across many chunks
    _check(*_case("bw_long", [1100], 1, 3, seed=8, alpha_mu=-6.0))


def test_backward_sixteen_heads_4k_packed():
    # a mid-size packed case with the benchmark's head layout on a quarter of the heads
    case, dO, dSf = _case("bw_4k", [1500, 2596], 4, 12, seed=9)
    _check(case, dO, dSf)


def test_backward_bench_layout():
    # 16/48 heads on one sequence: 48-column slices, where the forward re-run
    # saves its states from the tcgen05 state pass
    case, dO, dSf = _case("bw_48", [1000], 16, 48, seed=10)
    _check(case, dO, dSf)


def test_backward_two_sequences_64_column_slices():
    # 2 x 48 value-head units: 64-column slices, both chains on tcgen05
    case, dO, dSf = _case("bw_64", [300, 200], 16, 48, seed=12)
    _check(case, dO, dSf)


def test_backward_empty_sequence_64_column_slices():
    # an empty sequence between two others on the tcgen05 chains (3 x 48 units)
    case, dO, dSf = _case("bw_64_empty", [190, 0, 130], 16, 48, seed=14)
    _check(case, dO, dSf)


@pytest.mark.parametrize("lens,H_qk,H_v", [([100, 0, 37, 64], 2, 6), ([1100], 1, 3)])
def test_backward_fp32_io(lens, H_qk, H_v):
    # fp32 inputs and gradients (the products read bf16 copies of q, k, v and dO)
    case, dO, dSf = _case("bw_f32", lens, H_qk, H_v, seed=11, alpha_mu=-6.0,
                          dtype=torch.float32)
    _check(case, dO, dSf, dtype=torch.float32)


# (the last three: 48 value-head units, so 48-column slices, and 96 units, so
# 64-column slices; the tcgen05 state pass writes outputs and saved states
# together)
@pytest.mark.parametrize("lens,H_qk,H_v,dtype", [([100, 0, 37, 64], 2, 6, torch.bfloat16),
                                                 ([1100], 1, 3, torch.bfloat16),
                                                 ([300, 65], 2, 4, torch.float32),
                                                 ([700], 16, 48, torch.bfloat16),
                                                 ([333, 130], 8, 24, torch.float32),
                                                 ([250, 190], 16, 48, torch.bfloat16)])
def test_training_forward_then_saved_backward(lens, H_qk, H_v, dtype):
    # the training forward's outputs match the oracle's forward; the backward that
    # reads its saved states matches the oracle's gradients
    import oracle
    case, dO, dSf = _case("train", lens, H_qk, H_v, seed=13 + len(lens), alpha_mu=-3.0,
                          dtype=dtype)
    d = lambda x: None if x is None else x.cuda()
    o, S, ws = gdn.prefill_train(d(case.q), d(case.k), d(case.v), d(case.log_alpha),
                                 d(case.beta), S0=d(case.S0), cu_seqlens=d(case.cu_seqlens))
    torch.cuda.synchronize()
    assert o.dtype == dtype
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, S0=case.S0,
                                  cu_seqlens=case.cu_seqlens)
    assert np.abs(o.float().cpu().double().numpy() - o_ref).max() / np.abs(o_ref).max() <= TOL
    assert np.linalg.norm(S.cpu().double().numpy() - S_ref) / np.linalg.norm(S_ref) <= TOL
    got = gdn.prefill_backward(d(case.q), d(case.k), d(case.v), d(case.log_alpha), d(case.beta),
                               d(dO), S0=d(case.S0), dS_final=d(dSf),
                               cu_seqlens=d(case.cu_seqlens), workspace=ws, saved=True)
    torch.cuda.synchronize()
    assert gdn.last_device_error() == gdn.GDN_OK
    ref = backward.prefill_backward(case.q, case.k, case.v, case.log_alpha, case.beta,
                                    dO.float().numpy(),
                                    S0=None if case.S0 is None else case.S0.numpy(),
                                    dS_final=None if dSf is None else dSf.numpy(),
                                    cu_seqlens=case.cu_seqlens.numpy())
    for name, a, b in zip(["dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"], got, ref):
        a = a.float().cpu().double().numpy()
        err = np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)
        assert err <= TOL, (name, err)
