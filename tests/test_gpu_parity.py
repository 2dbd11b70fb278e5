"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small cases are compared element by element over every output; the full-size
workloads (in the launch configuration the benchmark times) are compared on
sampled value heads / (sequence, head) units that the oracle computes one by
one.  Tolerances are the acceptance bar in tests/gpu_util.py.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_12_b200 import gdn, inputs
from tests.gpu_util import (O_TOL, S_TOL, o_err, per_head_o, per_head_s, record, s_err,
                            to_cuda)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert gdn.last_device_error() == gdn.GDN_OK


def _run_case(case, heads=None, want_o=True, state=True):
    c = to_cuda(case)
    o, S = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"],
                       cu_seqlens=c["cu_seqlens"], want_state=state)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, S0=case.S0,
                                  cu_seqlens=case.cu_seqlens, heads=heads, want_o=want_o)
    return o, S, o_ref, S_ref


# ------------------------------------------------------------------ decode
def _decode_check(B, H_qk, H_v, dtype, seed, steps=3):
    dc = inputs.make_decode(B, H_qk, H_v, 128, seed=seed)
    S = dc.S0.cuda()
    S_ref = dc.S0.double().numpy()
    for s in range(steps):
        q, k, v, la, be = dc.step(s, dtype)
        o = gdn.decode_step(q.cuda(), k.cuda(), v.cuda(), la.cuda(), be.cuda(), S)
        o_ref, S_ref = oracle.decode_step(q, k, v, la, be, S_ref)
        assert o_err(o, o_ref) <= O_TOL
        assert s_err(S, S_ref) <= S_TOL


@pytest.mark.parametrize("B,H_qk,H_v,dtype", [(3, 2, 6, torch.bfloat16), (2, 1, 1, torch.float32),
                                               (5, 4, 4, torch.bfloat16)])
def test_decode_small(B, H_qk, H_v, dtype):
    _decode_check(B, H_qk, H_v, dtype, seed=B * 10 + H_v)


def test_decode_batched_256_full_512_steps_sampled():
    """The batched-decode workload (256 sequences, 16/48 heads, 512 steps):
    every step runs on the full state in place; o is checked at every step and
    S after step 512 on 24 sampled (sequence, head) units."""
    dc = inputs.batched_decode_256()
    S = dc.S0.cuda()
    rng = np.random.default_rng(0)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, 256, 24), rng.integers(0, 48, 24))]
    S_ref = np.stack([dc.S0[b, h].double().numpy() for b, h in pairs])
    worst_o = 0.0
    for s in range(512):
        q, k, v, la, be = dc.step(s)
        o = gdn.decode_step(q.cuda(), k.cuda(), v.cuda(), la.cuda(), be.cuda(), S)
        o_ref, S_ref = oracle.decode_step(q, k, v, la, be, S_ref, units_bh=pairs)
        og = o.float().cpu().numpy()
        worst_o = max(worst_o, o_err(np.stack([og[b, h] for b, h in pairs]), o_ref))
    Sg = S.cpu().double().numpy()
    se = s_err(np.stack([Sg[b, h] for b, h in pairs]), S_ref)
    record("decode_batched_256", "batched decode: 256 sequences x 16/48 heads, 512 steps", o_err=worst_o,
           s_err=se, units="24 sampled (sequence, head) units")
    assert worst_o <= O_TOL
    assert se <= S_TOL


# ------------------------------------------------------------------ prefill, small
def test_prefill_tiny_fp32_L256():
    """B=1, L=256, 1 QK / 1 V head, d=128, all fp32, S0=0, seed 0."""
    case = inputs.tiny_fp32()
    o, S, o_ref, S_ref = _run_case(case)
    assert o.dtype == torch.float32
    oe, se = o_err(o, o_ref), s_err(S, S_ref)
    record("prefill_tiny_fp32_L256", "tiny prefill: L=256, 1/1 heads, fp32", o_err=oe, s_err=se)
    assert oe <= O_TOL
    assert se <= S_TOL


@pytest.mark.parametrize("lens", [[1], [63], [64], [65], [200], [17, 64, 1, 0, 130], [0]])
@pytest.mark.parametrize("s0", [False, True])
def test_prefill_ragged_small(lens, s0):
    case = inputs.make_prefill("small", lens, 2, 6, seed=sum(lens) + 7 * s0, s0=s0)
    o, S, o_ref, S_ref = _run_case(case)
    if case.T:
        assert o_err(o, o_ref) <= O_TOL
    assert s_err(S, S_ref) <= S_TOL if np.abs(S_ref).max() > 0 else np.abs(S.cpu().numpy()).max() == 0


@pytest.mark.parametrize("H_qk,H_v", [(1, 1), (1, 3), (4, 4), (16, 48)])
def test_prefill_head_layouts(H_qk, H_v):
    case = inputs.make_prefill("heads", [300], H_qk, H_v, seed=H_qk * 100 + H_v, s0=True)
    heads = None if H_v <= 6 else [0, 1, 2, 23, 47]
    o, S, o_ref, S_ref = _run_case(case, heads=heads)
    hs = list(range(H_v)) if heads is None else heads
    assert o_err(o[:, hs], o_ref[:, hs]) <= O_TOL
    assert s_err(S[:, hs], S_ref[:, hs]) <= S_TOL


def test_prefill_fp32_io_ragged():
    case = inputs.make_prefill("f32", [77, 150], 2, 4, dtype=torch.float32, seed=5, s0=True)
    o, S, o_ref, S_ref = _run_case(case)
    assert o_err(o, o_ref) <= O_TOL
    assert s_err(S, S_ref) <= S_TOL


def test_prefill_without_state_output():
    case = inputs.make_prefill("nostate", [130], 1, 3, seed=3)
    o, S, o_ref, _ = _run_case(case, state=False)
    assert S is None
    assert o_err(o, o_ref) <= O_TOL


# ------------------------------------------------------------------ self-consistency
def test_prefill_equals_repeated_decode():
    case = inputs.make_prefill("pd", [37], 2, 6, seed=11, s0=True)
    c = to_cuda(case)
    o_p, S_p = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"])
    S = c["S0"].clone()
    outs = []
    for t in range(37):
        outs.append(gdn.decode_step(c["q"][t:t + 1], c["k"][t:t + 1], c["v"][t:t + 1],
                                    c["log_alpha"][t:t + 1], c["beta"][t:t + 1], S)[0])
    o_d = torch.stack(outs)
    assert o_err(o_p, o_d.float().cpu().double().numpy()) <= O_TOL
    assert s_err(S_p, S.cpu().double().numpy()) <= S_TOL


@pytest.mark.parametrize("m", [64, 100])
def test_split_sequence_via_S0_in_place(m):
    """prefill(x[:m]) -> S_m, then prefill(x[m:], S0=S_m) with S_final aliasing
    S0 (in place) equals prefill(x)."""
    case = inputs.make_prefill("split", [230], 2, 6, seed=m, s0=True)
    c = to_cuda(case)
    o, S = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"])
    oa, Sa = gdn.prefill(c["q"][:m], c["k"][:m], c["v"][:m], c["log_alpha"][:m], c["beta"][:m],
                         S0=c["S0"])
    ob, _ = gdn.prefill(c["q"][m:].contiguous(), c["k"][m:].contiguous(), c["v"][m:].contiguous(),
                        c["log_alpha"][m:].contiguous(), c["beta"][m:].contiguous(), S0=Sa,
                        S_final=Sa)
    o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, S0=case.S0)
    assert o_err(torch.cat([oa, ob]), o_ref) <= O_TOL
    assert s_err(Sa, S_ref) <= S_TOL
    assert s_err(S, S_ref) <= S_TOL


def test_gqa_equals_replicated_heads():
    case = inputs.make_prefill("gqa", [150], 2, 6, seed=21, s0=True)
    c = to_cuda(case)
    o1, S1 = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"])
    qr = c["q"].repeat_interleave(3, dim=1).contiguous()
    kr = c["k"].repeat_interleave(3, dim=1).contiguous()
    o2, S2 = gdn.prefill(qr, kr, c["v"], c["log_alpha"], c["beta"], S0=c["S0"])
    assert torch.equal(o1, o2)
    assert torch.equal(S1, S2)


def test_packed_varlen_equals_separate_calls():
    case = inputs.make_prefill("pack", [70, 1, 128, 33], 2, 6, seed=8, s0=True)
    c = to_cuda(case)
    o, S = gdn.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], S0=c["S0"],
                       cu_seqlens=c["cu_seqlens"])
    cu = case.cu_seqlens.tolist()
    for n in range(4):
        sl = slice(cu[n], cu[n + 1])
        on, Sn = gdn.prefill(c["q"][sl], c["k"][sl], c["v"][sl], c["log_alpha"][sl].contiguous(),
                             c["beta"][sl].contiguous(), S0=c["S0"][n:n + 1].contiguous())
        assert torch.equal(o[sl], on)
        assert torch.equal(S[n:n + 1], Sn)


# ------------------------------------------------------------------ full-size workloads
def test_prefill_qwen_32k_sampled_heads():
    """B=1, L=32768, 16 QK / 48 V heads, bf16 q/k/v (the benchmarked launch)."""
    case = inputs.qwen_prefill_32k()
    heads = [0, 25, 47]
    o, S, o_ref, S_ref = _run_case(case, heads=heads)
    oe, se = o_err(o[:, heads], o_ref[:, heads]), s_err(S[:, heads], S_ref[:, heads])
    record("prefill_qwen_32k", "prefill L=32768, 16/48 heads, bf16", o_err=oe, s_err=se,
           o_per_head=per_head_o(o, o_ref, heads), s_per_head=per_head_s(S, S_ref, heads))
    assert oe <= O_TOL
    assert se <= S_TOL
    assert torch.isfinite(o.float()).all()


def test_prefill_varlen_8seq_sampled_heads():
    case = inputs.varlen_8seq()
    heads = [5, 40]
    o, S, o_ref, S_ref = _run_case(case, heads=heads)
    oe, se = o_err(o[:, heads], o_ref[:, heads]), s_err(S[:, heads], S_ref[:, heads])
    record("prefill_varlen_8seq", "packed varlen prefill: 8 sequences of 1024-8192, S0 != 0", o_err=oe, s_err=se,
           o_per_head=per_head_o(o, o_ref, heads), s_per_head=per_head_s(S, S_ref, heads))
    assert oe <= O_TOL
    assert se <= S_TOL


@pytest.mark.slow
def test_prefill_long_256k_final_state_sampled_heads():
    """L=262144 with long-memory gates: S_final checked on sampled heads."""
    case = inputs.long_256k()
    heads = [7, 31]
    o, S, o_ref, S_ref = _run_case(case, heads=heads, want_o=False)
    se = s_err(S[:, heads], S_ref[:, heads])
    record("prefill_long_256k", "long-context prefill: L=262144, long-memory gates", s_err=se,
           s_per_head=per_head_s(S, S_ref, heads))
    assert se <= S_TOL
    assert torch.isfinite(o.float()).all()


def test_prefill_long_memory_gates_bench_layout_sampled_heads():
    """Gates that remember across many chunks (log_alpha = -softplus(N(-6, 1)),
    alpha ~ 0.9975 per token) at the benchmark's head layout (16/48 heads,
    48-column slices of the state), 8192 tokens: o and S on sampled heads."""
    case = inputs.make_prefill("longmem_bench_layout", [8192], 16, 48, seed=12, alpha_mu=-6.0)
    heads = [1, 22, 46]
    o, S, o_ref, S_ref = _run_case(case, heads=heads)
    oe, se = o_err(o[:, heads], o_ref[:, heads]), s_err(S[:, heads], S_ref[:, heads])
    record("prefill_longmem_bench_layout", "L=8192, 16/48 heads, log_alpha=-softplus(N(-6,1))",
           o_err=oe, s_err=se, o_per_head=per_head_o(o, o_ref, heads),
           s_per_head=per_head_s(S, S_ref, heads))
    assert oe <= O_TOL
    assert se <= S_TOL
