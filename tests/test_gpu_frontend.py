"""Parity of the front end (gdn_frontend, gdn_frontend_decode_step) with the
fp64 oracle (oracle/frontend.py), and of the front end followed by the
prefill with the oracle's front end followed by the oracle's recurrence."""
import numpy as np
import pytest
import torch

import oracle
from oracle import frontend as fe
from linear_attention_12_b200 import gdn, inputs
from tests.gpu_util import O_TOL, S_TOL, o_err, s_err

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert gdn.last_device_error() == gdn.GDN_OK


def _rel(a, b, mask=None):
    a = a.float().cpu().double().numpy() if isinstance(a, torch.Tensor) else a
    b = b.float().cpu().double().numpy() if isinstance(b, torch.Tensor) else b
    b = np.asarray(b, dtype=np.float64)
    if mask is not None:
        a, b = a[mask], b[mask]
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def _cuda(case):
    return dict(q_raw=case.q_raw.cuda(), k_raw=case.k_raw.cuda(), v_raw=case.v_raw.cuda(),
                conv_w=case.conv_w.cuda(), a=case.a.cuda(), b=case.b.cuda(),
                cu_seqlens=case.cu_seqlens.cuda())


# bf16 outputs carry one bf16 rounding (relative 2^-9); fp32 outputs fp32 arithmetic
TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-5}


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("act", ["none", "silu"])
def test_frontend_packed_small(dtype, act):
    case = inputs.make_frontend("fe_small", [1, 5, 64, 100, 0, 37], 2, 6, dtype=dtype, seed=21)
    c = _cuda(case)
    q, k, v, la, be = gdn.frontend(**c, act=act, eps=1e-6)
    torch.cuda.synchronize()
    rq, rk, rv, rla, rbe = fe.frontend(case.q_raw, case.k_raw, case.v_raw, case.conv_w, case.a,
                                       case.b, case.cu_seqlens, act=act, eps=1e-6)
    for x, y in ((q, rq), (k, rk), (v, rv)):
        assert _rel(x, y) <= TOL[dtype]
    assert _rel(la, rla) <= 1e-6
    assert _rel(be, rbe) <= 1e-6
    qn = q.float().norm(dim=-1)
    assert torch.allclose(qn, torch.ones_like(qn), atol=1e-2)


def test_frontend_full_size_sampled_rows():
    """L=32768, 16/48 heads, bf16: every row the oracle evaluates on its own."""
    case = inputs.make_frontend("fe_32k", [32768], 16, 48, seed=22)
    c = _cuda(case)
    q, k, v, la, be = gdn.frontend(**c, act="silu")
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 1, 2, 3, 63, 64, 65, 32767], rng.integers(0, 32768, 40)]))
    rq, rk, rv, rla, rbe = fe.frontend(case.q_raw, case.k_raw, case.v_raw, case.conv_w, case.a,
                                       case.b, case.cu_seqlens, act="silu", rows=rows)
    ridx = torch.from_numpy(rows).cuda()
    for x, y in ((q, rq), (k, rk), (v, rv), (la, rla), (be, rbe)):
        assert _rel(x[ridx], y) <= 1e-2


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_frontend_decode_steps(dtype):
    """Decode steps with the ring state equal the oracle's decode steps, and the
    GPU's own prefill front end on the same tokens."""
    B, H_qk, H_v, steps = 3, 2, 6, 6
    case = inputs.make_frontend("fe_dec", [steps] * B, H_qk, H_v, dtype=dtype, seed=23)
    C = (2 * H_qk + H_v) * 128
    state = torch.zeros((B, 3, C), dtype=dtype, device="cuda")
    ref_state = np.zeros((B, 3, C))
    pre = gdn.frontend(**_cuda(case), act="silu")
    w = case.conv_w.cuda()
    for s in range(steps):
        idx = torch.arange(B) * steps + s  # token s of every sequence
        args = [case.q_raw[idx], case.k_raw[idx], case.v_raw[idx]]
        out = gdn.frontend_decode_step(*[t.cuda() for t in args], w, case.a[idx].cuda(),
                                       case.b[idx].cuda(), state, act="silu")
        torch.cuda.synchronize()
        ref = fe.frontend_decode_step(*args, case.conv_w, case.a[idx], case.b[idx], ref_state,
                                      act="silu")
        ref_state = ref[5]
        for x, y, z in zip(out, ref[:5], pre):
            assert _rel(x, y) <= TOL[dtype]
            assert _rel(x, z[idx.cuda()].cpu()) <= TOL[dtype]
    assert _rel(state.cpu(), ref_state) == 0.0  # raw rows are kept exactly


def test_frontend_then_prefill_matches_oracle_pipeline():
    case = inputs.make_frontend("fe_pipe", [150, 77], 2, 6, seed=24)
    c = _cuda(case)
    q, k, v, la, be = gdn.frontend(**c, act="silu")
    o, S = gdn.prefill(q, k, v, la, be, cu_seqlens=c["cu_seqlens"])
    torch.cuda.synchronize()
    rq, rk, rv, rla, rbe = fe.frontend(case.q_raw, case.k_raw, case.v_raw, case.conv_w, case.a,
                                       case.b, case.cu_seqlens, act="silu")
    # the oracle recurrence on the oracle's front end (fp32 inputs, the exact values)
    o_ref, S_ref = oracle.prefill(rq.astype(np.float32), rk.astype(np.float32),
                                  rv.astype(np.float32), rla.astype(np.float32),
                                  rbe.astype(np.float32), cu_seqlens=case.cu_seqlens)
    assert o_err(o, o_ref) <= O_TOL
    assert s_err(S, S_ref) <= S_TOL
