"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every symbol the header declares, and rejects invalid arguments on the host
before any CUDA call."""
import ctypes
import os
import re

import pytest

from linear_attention_12_b200 import build as gdn_build
from linear_attention_12_b200 import gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    gdn_build.build()
    return gdn.lib()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "gdn.h")).read()
    return set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text))


def test_header_declares_expected_entry_points():
    assert {"gdn_prefill", "gdn_prefill_workspace_size", "gdn_decode_step",
            "gdn_get_last_device_error", "gdn_status_string", "gdn_version"} <= _declared_symbols()


def test_library_exports_every_declared_symbol(L):
    for name in _declared_symbols():
        assert hasattr(L, name), name
    assert set(gdn.SIGNATURES) == _declared_symbols()


def test_status_strings(L):
    for code, name in [(0, "GDN_OK"), (1, "GDN_ERR_INVALID_ARG"), (2, "GDN_ERR_UNSUPPORTED"),
                       (3, "GDN_ERR_CUDA"), (4, "GDN_ERR_TIMEOUT"), (5, "GDN_ERR_WORKSPACE")]:
        assert gdn.status_string(code) == name
    assert L.gdn_version() == 100


REC_BYTES = 2 * 64 * 64 * 2 + 132 * 4  # per (chunk slot, value head): two bf16 tiles + vectors


def test_workspace_size(L):
    # one chunk-operator record per (chunk slot, value head); slots = N + ceil(T / 64)
    ws = gdn.workspace_size(1, 32768, 16, 48, 128, gdn.GDN_BF16)
    assert ws >= (1 + 512) * 48 * REC_BYTES
    assert ws < (1 + 512) * 48 * REC_BYTES + 256
    ws32 = gdn.workspace_size(1, 256, 1, 1, 128, gdn.GDN_F32)
    assert ws32 >= 3 * 256 * 128 * 2 + (1 + 4) * REC_BYTES  # + bf16 copies of q, k, v
    assert gdn.workspace_size(3, 0, 1, 1, 128, gdn.GDN_BF16) == 0  # nothing to do
    assert gdn.workspace_size(0, 256, 1, 1, 128, gdn.GDN_F32) == 0  # invalid -> 0


# Fake, never dereferenced device addresses: validation fails before any use.
P = 0x10000
BAD = 0x10001  # misaligned


def _prefill(L, **kw):
    a = dict(q=P, k=P, v=P, la=P, be=P, S0=None, cu=P, N=1, T=64, H_qk=1, H_v=1, dk=128,
             dv=128, dt=gdn.GDN_BF16, o=P, Sf=None, ws=None, wsb=0, stream=None)
    a.update(kw)
    return L.gdn_prefill(a["q"], a["k"], a["v"], a["la"], a["be"], a["S0"], a["cu"], a["N"],
                         a["T"], a["H_qk"], a["H_v"], a["dk"], a["dv"], a["dt"], a["o"], a["Sf"],
                         a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(o=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(cu=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(v=BAD), gdn.GDN_ERR_INVALID_ARG),
    (dict(S0=BAD), gdn.GDN_ERR_INVALID_ARG),
    (dict(H_qk=3, H_v=4), gdn.GDN_ERR_INVALID_ARG),
    (dict(H_qk=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(T=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(dt=7), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=64, dv=64), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dv=256), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dt=gdn.GDN_F32), gdn.GDN_ERR_WORKSPACE),
    (dict(dt=gdn.GDN_F32, ws=P, wsb=16), gdn.GDN_ERR_WORKSPACE),
])
def test_prefill_rejects_bad_arguments_on_host(L, kw, expect):
    assert _prefill(L, **kw) == expect


@pytest.mark.parametrize("entry", ["gdn_prefill_tc", "gdn_prefill_mma"])
@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(H_qk=3, H_v=4), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=64, dv=64), gdn.GDN_ERR_UNSUPPORTED),
    (dict(wsb=16), gdn.GDN_ERR_WORKSPACE),
    (dict(), gdn.GDN_ERR_CUDA),  # host checks pass; no device here
])
def test_fixed_state_pass_entries_check_like_the_prefill(L, entry, kw, expect):
    a = dict(q=P, k=P, v=P, la=P, be=P, S0=None, cu=P, N=1, T=64, H_qk=1, H_v=1, dk=128,
             dv=128, dt=gdn.GDN_BF16, o=P, Sf=None, ws=P, wsb=1 << 40, stream=None)
    a.update(kw)
    assert getattr(L, entry)(*a.values()) == expect


def _prefill_seg(L, segments, **kw):
    a = dict(q=P, k=P, v=P, la=P, be=P, S0=None, cu=P, N=1, T=4096, H_qk=1, H_v=1, dk=128,
             dv=128, dt=gdn.GDN_BF16, o=P, Sf=None, ws=P, wsb=1 << 40, stream=None)
    a.update(kw)
    return L.gdn_prefill_segmented(a["q"], a["k"], a["v"], a["la"], a["be"], a["S0"], a["cu"],
                                   a["N"], a["T"], a["H_qk"], a["H_v"], a["dk"], a["dv"], a["dt"],
                                   a["o"], a["Sf"], segments, a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("segments", [-1, 65])
def test_segmented_prefill_rejects_segment_counts_out_of_range(L, segments):
    assert _prefill_seg(L, segments) == gdn.GDN_ERR_INVALID_ARG


def test_segmented_prefill_checks_its_workspace(L):
    need = L.gdn_prefill_segmented_workspace_size(1, 4096, 1, 1, 128, 128, gdn.GDN_BF16, 4)
    assert _prefill_seg(L, 4, wsb=need - 1) == gdn.GDN_ERR_WORKSPACE
    assert _prefill_seg(L, 4, ws=P + 16, wsb=need) == gdn.GDN_ERR_WORKSPACE  # not 256-aligned


def test_segmented_workspace_adds_the_pieces_states(L):
    ws = lambda seg: L.gdn_prefill_segmented_workspace_size(1, 32768, 2, 6, 128, 128,
                                                            gdn.GDN_BF16, seg)
    one, four = ws(1), ws(4)
    rec = 16912 * 6  # one more record slot per extra piece, per value head
    states = 3 * 4 * 6 * 128 * 128 * 4  # R, P_s and the entering state of every piece
    assert four - one >= 3 * rec + states
    assert four - one <= 3 * rec + states + 4 * 256 + 256  # plus the piece starts and rounding
    assert ws(0) == ws(L.gdn_prefill_auto_segments(1, 32768, 2, 6))
    assert L.gdn_prefill_segmented_workspace_size(1, 32768, 2, 6, 128, 128, gdn.GDN_BF16, 65) == 0


def test_automatic_split_only_for_few_chains(L):
    assert L.gdn_prefill_auto_segments(1, 32768, 16, 48) == 1   # 48 heads fill the SMs
    assert L.gdn_prefill_auto_segments(8, 65536, 16, 48) == 1
    assert L.gdn_prefill_auto_segments(1, 256, 1, 1) == 1        # too short to split
    assert L.gdn_prefill_auto_segments(1, 32768, 2, 6) > 1       # a tensor-parallel shard
    assert L.gdn_prefill_auto_segments(1, 32768, 1, 1) > 1
    assert L.gdn_prefill_auto_segments(0, 32768, 1, 1) == 1      # invalid: no split


def _backward(L, **kw):
    a = dict(q=P, k=P, v=P, la=P, be=P, S0=None, cu=P, dO=P, dSf=None, N=1, T=64, H_qk=1, H_v=1,
             dk=128, dv=128, dt=gdn.GDN_BF16, dq=P, dk_out=P, dv_out=P, dla=P, dbe=P, dS0=None,
             ws=P, wsb=1 << 40, stream=None)
    a.update(kw)
    return L.gdn_prefill_backward(a["q"], a["k"], a["v"], a["la"], a["be"], a["S0"], a["cu"],
                                  a["dO"], a["dSf"], a["N"], a["T"], a["H_qk"], a["H_v"], a["dk"],
                                  a["dv"], a["dt"], a["dq"], a["dk_out"], a["dv_out"], a["dla"],
                                  a["dbe"], a["dS0"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,expect", [
    (dict(dO=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dq=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dv_out=P + 8), gdn.GDN_ERR_INVALID_ARG),
    (dict(dla=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dS0=BAD), gdn.GDN_ERR_INVALID_ARG),
    (dict(wsb=16), gdn.GDN_ERR_WORKSPACE),
    (dict(ws=P + 64), gdn.GDN_ERR_WORKSPACE),   # not 256-byte aligned
    (dict(H_qk=2, H_v=3), gdn.GDN_ERR_INVALID_ARG),
])
def test_backward_rejects_bad_arguments_on_host(L, kw, expect):
    assert _backward(L, **kw) == expect


def test_backward_fp32_needs_room_for_bf16_copies(L):
    ws16 = L.gdn_prefill_backward_workspace_size(1, 64, 1, 1, 128, 128, gdn.GDN_BF16)
    ws32 = L.gdn_prefill_backward_workspace_size(1, 64, 1, 1, 128, 128, gdn.GDN_F32)
    assert ws32 > ws16
    assert _backward(L, dt=gdn.GDN_F32, wsb=ws16) == gdn.GDN_ERR_WORKSPACE
    assert _backward(L, dt=gdn.GDN_BF16, wsb=ws16) == gdn.GDN_ERR_CUDA  # host checks pass; no device


def test_training_forward_checks_its_workspace(L):
    ws = L.gdn_prefill_backward_workspace_size(1, 64, 1, 1, 128, 128, gdn.GDN_BF16)
    args = lambda wsb, dt=gdn.GDN_BF16, o=P: (P, P, P, P, P, None, P, 1, 64, 1, 1, 128, 128, dt,
                                                o, None, P, wsb, None)
    assert L.gdn_prefill_train(*args(ws - 256)) == gdn.GDN_ERR_WORKSPACE
    assert L.gdn_prefill_train(*args(ws, gdn.GDN_F32)) == gdn.GDN_ERR_WORKSPACE  # + bf16 copies
    assert L.gdn_prefill_train(*args(ws, o=None)) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_prefill_train(*args(ws)) == gdn.GDN_ERR_CUDA  # host checks pass; no device
    assert _backward(L, wsb=16) == gdn.GDN_ERR_WORKSPACE
    b = dict(q=P, k=P, v=P, la=P, be=P, S0=None, cu=P, dO=P, dSf=None, N=1, T=64, H_qk=1, H_v=1,
             dk=128, dv=128, dt=gdn.GDN_BF16, dq=P, dk_out=P, dv_out=P, dla=P, dbe=P, dS0=None,
             ws=P, wsb=16, stream=None)
    assert L.gdn_prefill_backward_saved(*b.values()) == gdn.GDN_ERR_WORKSPACE


def test_backward_workspace_holds_records_and_two_states_per_chunk(L):
    # per (chunk slot, value head): the 16,912-byte record and two bf16 state images
    N, T, H_v = 1, 4096, 3
    ws = L.gdn_prefill_backward_workspace_size(N, T, 1, H_v, 128, 128, gdn.GDN_BF16)
    slots = N + T // 64
    assert ws >= slots * H_v * (16912 + 2 * 128 * 128 * 2)
    assert ws <= slots * H_v * (16912 + 2 * 128 * 128 * 2) + 3 * 256
    # fp32 I/O adds bf16 copies of q, k (1 head) and v, dO (H_v heads)
    ws32 = L.gdn_prefill_backward_workspace_size(N, T, 1, H_v, 128, 128, gdn.GDN_F32)
    assert ws32 == ws + 2 * T * 128 * 2 * (1 + H_v)


def _decode(L, **kw):
    a = dict(q=P, k=P, v=P, la=P, be=P, S=P, B=4, H_qk=1, H_v=3, dk=128, dv=128,
             dt=gdn.GDN_BF16, o=P, stream=None)
    a.update(kw)
    return L.gdn_decode_step(a["q"], a["k"], a["v"], a["la"], a["be"], a["S"], a["B"], a["H_qk"],
                             a["H_v"], a["dk"], a["dv"], a["dt"], a["o"], a["stream"])


@pytest.mark.parametrize("kw,expect", [
    (dict(S=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(S=BAD), gdn.GDN_ERR_INVALID_ARG),
    (dict(q=P + 8), gdn.GDN_ERR_INVALID_ARG),
    (dict(B=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(H_qk=2, H_v=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(B=0, q=None, S=None), gdn.GDN_OK),  # nothing to do, nothing touched
])
def test_decode_rejects_bad_arguments_on_host(L, kw, expect):
    assert _decode(L, **kw) == expect


def _decode_multi(L, **kw):
    a = dict(q=P, k=P, v=P, la=P, be=P, S=P, B=4, M=4, H_qk=1, H_v=3, dk=128, dv=128,
             dt=gdn.GDN_BF16, o=P, Ss=P + (1 << 30), stream=None)
    a.update(kw)
    return L.gdn_decode_multi(a["q"], a["k"], a["v"], a["la"], a["be"], a["S"], a["B"], a["M"],
                              a["H_qk"], a["H_v"], a["dk"], a["dv"], a["dt"], a["o"], a["Ss"],
                              a["stream"])


_STATE = 3 * 128 * 128 * 4  # bytes of one sequence's states at H_v = 3


@pytest.mark.parametrize("kw,expect", [
    (dict(M=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(M=9), gdn.GDN_ERR_INVALID_ARG),   # above GDN_MAX_DECODE_TOKENS
    (dict(Ss=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(Ss=P + 8), gdn.GDN_ERR_INVALID_ARG),
    (dict(S=BAD), gdn.GDN_ERR_INVALID_ARG),
    (dict(B=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(Ss=P), gdn.GDN_ERR_INVALID_ARG),                      # checkpoints over the input
    (dict(Ss=P + 4 * _STATE - 16 * 1024), gdn.GDN_ERR_INVALID_ARG),  # partial overlap
    (dict(M=1, Ss=P + _STATE), gdn.GDN_ERR_INVALID_ARG),        # M = 1, shifted: overlap
    (dict(H_qk=2, H_v=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(dv=64), gdn.GDN_ERR_UNSUPPORTED),
    (dict(B=0, q=None, S=None, Ss=None), gdn.GDN_OK),  # nothing to do, nothing touched
])
def test_decode_multi_rejects_bad_arguments_on_host(L, kw, expect):
    assert _decode_multi(L, **kw) == expect


def test_binding_refuses_cpu_tensors(L):
    import torch
    x = torch.zeros(4, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        gdn.decode_step(x, x, x, torch.zeros(4, 1), torch.zeros(4, 1), torch.zeros(4, 1, 128, 128))


def test_binding_has_no_cpu_fallback():
    """The product binding must not reach the oracle or any CPU path."""
    src = open(os.path.join(ROOT, "linear_attention_12_b200", "gdn.py")).read()
    assert "oracle" not in src
    assert "import numpy" not in src


def test_noalloc_rejects_scratch_beyond_its_maximum_on_host(L):
    """The no-allocation prefill refuses, before any CUDA call, a call whose
    scratch would exceed its fixed array."""
    cap = L.gdn_prefill_noalloc_max_scratch_bytes()
    assert cap == 16 << 20
    T = cap // ((2 * 16 + 48) * 128 * 2) + 64
    st = L.gdn_prefill_noalloc(P, P, P, P, P, None, P, 1, T, 16, 48, 128, 128, gdn.GDN_F32,
                               P, None, None)
    assert st == gdn.GDN_ERR_WORKSPACE
    # invalid arguments are still rejected by the prefill's own checks
    st = L.gdn_prefill_noalloc(None, P, P, P, P, None, P, 1, 64, 1, 1, 128, 128, gdn.GDN_BF16,
                               P, None, None)
    assert st == gdn.GDN_ERR_INVALID_ARG


def _frontend(L, **kw):
    a = dict(q=P, k=P, v=P, w=P, a=P, b=P, cu=P, N=1, T=64, H_qk=1, H_v=3, dk=128, dv=128,
             dt=gdn.GDN_BF16, act=gdn.GDN_ACT_NONE, eps=1e-6, oq=P, ok=P, ov=P, la=P, be=P,
             stream=None)
    a.update(kw)
    return L.gdn_frontend(a["q"], a["k"], a["v"], a["w"], a["a"], a["b"], a["cu"], a["N"],
                          a["T"], a["H_qk"], a["H_v"], a["dk"], a["dv"], a["dt"], a["act"],
                          a["eps"], a["oq"], a["ok"], a["ov"], a["la"], a["be"], a["stream"])


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(w=P + 4), gdn.GDN_ERR_INVALID_ARG),   # the weight is read as float4
    (dict(ov=BAD), gdn.GDN_ERR_INVALID_ARG),
    (dict(la=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(act=2), gdn.GDN_ERR_INVALID_ARG),
    (dict(eps=-1.0), gdn.GDN_ERR_INVALID_ARG),
    (dict(eps=float("nan")), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(H_qk=2, H_v=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=64, dv=64), gdn.GDN_ERR_UNSUPPORTED),
])
def test_frontend_rejects_bad_arguments_on_host(L, kw, expect):
    assert _frontend(L, **kw) == expect


def test_frontend_decode_rejects_bad_arguments_on_host(L):
    def call(**kw):
        a = dict(q=P, k=P, v=P, w=P, a=P, b=P, st=P, B=2, H_qk=1, H_v=3, dk=128, dv=128,
                 dt=gdn.GDN_BF16, act=gdn.GDN_ACT_SILU, eps=0.0, oq=P, ok=P, ov=P, la=P, be=P)
        a.update(kw)
        return L.gdn_frontend_decode_step(a["q"], a["k"], a["v"], a["w"], a["a"], a["b"],
                                          a["st"], a["B"], a["H_qk"], a["H_v"], a["dk"], a["dv"],
                                          a["dt"], a["act"], a["eps"], a["oq"], a["ok"], a["ov"],
                                          a["la"], a["be"], None)
    assert call(st=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(st=BAD) == gdn.GDN_ERR_INVALID_ARG
    assert call(B=-1) == gdn.GDN_ERR_INVALID_ARG
    assert call(act=7) == gdn.GDN_ERR_INVALID_ARG
    assert call(B=0, q=None, st=None) == gdn.GDN_OK  # nothing to do, nothing touched
