"""Pins of the oracle's multi-token decode (oracle.decode_multi), the
speculative-verification form of the recurrence: checkpoints against the
explicit-matrix evaluation of the state-update formula (numpy, independent of
the C oracle), and two closed forms.  CPU only."""
import numpy as np
import torch

import oracle
from linear_attention_12_b200 import inputs


def _window(B, H_qk, H_v, d, M, seed):
    dc = inputs.make_decode(B, H_qk, H_v, d, seed=seed)
    return dc.S0, dc.window(0, M)


def test_checkpoints_equal_the_literal_formula_on_each_prefix():
    B, H_qk, H_v, d, M = 3, 1, 2, 8, 4
    S0, (q, k, v, la, be) = _window(B, H_qk, H_v, d, M, seed=21)
    o, S_steps = oracle.decode_multi(q, k, v, la, be, S0)
    assert o.shape == (B, M, H_v, d) and S_steps.shape == (B, M, H_v, d, d)
    for j in range(M):
        # prefix of j + 1 tokens of every sequence, packed, from the same S0
        n = j + 1
        cu = torch.arange(0, B * n + 1, n, dtype=torch.int32)
        flat = [x[:, :n].reshape(B * n, *x.shape[2:]) for x in (q, k, v, la, be)]
        o_lit, S_lit = oracle.literal_prefill(*flat, S0=S0, cu_seqlens=cu)
        np.testing.assert_allclose(S_steps[:, j], S_lit, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(o[:, j], o_lit.reshape(B, n, H_v, d)[:, j], rtol=1e-12,
                                   atol=1e-14)


def test_no_write_is_pure_decay():
    # beta = 0: S_j = exp(sum_{i<=j} log_alpha_i) S0 and o_j = S_j^T q_j
    B, H_qk, H_v, d, M = 2, 1, 3, 16, 4
    S0, (q, k, v, la, be) = _window(B, H_qk, H_v, d, M, seed=22)
    be = torch.zeros_like(be)
    o, S_steps = oracle.decode_multi(q, k, v, la, be, S0)
    g = np.cumsum(la.double().numpy(), axis=1)                       # [B, M, H_v]
    S_ref = np.exp(g)[..., None, None] * S0.double().numpy()[:, None]  # [B, M, H_v, d, d]
    np.testing.assert_allclose(S_steps, S_ref, rtol=1e-13, atol=0)
    qd = oracle._widen(q)                                            # [B, M, H_qk, d]
    grp = H_v // H_qk
    for h in range(H_v):
        o_ref = np.einsum("bmkv,bmk->bmv", S_ref[:, :, h], qd[:, :, h // grp])
        np.testing.assert_allclose(o[:, :, h], o_ref, rtol=1e-12, atol=1e-14)


def test_full_write_with_a_repeated_unit_key_keeps_the_last_value():
    # alpha = beta = 1 and the same unit key every token: each step replaces what
    # the memory returns for k with the new v, so S_j^T k = v_j exactly
    B, H_qk, H_v, d, M = 2, 1, 2, 8, 4
    S0, (q, k, v, la, be) = _window(B, H_qk, H_v, d, M, seed=23)
    k = torch.zeros_like(k)
    k[..., 0] = 1.0                       # e_0, exact in bf16
    la = torch.zeros_like(la)
    be = torch.ones_like(be)
    _, S_steps = oracle.decode_multi(q, k, v, la, be, S0)
    vd = oracle._widen(v)
    for j in range(M):
        np.testing.assert_allclose(S_steps[:, j, :, 0, :], vd[:, j], rtol=0, atol=1e-15)
        # the other key rows are untouched by a write along e_0
        np.testing.assert_array_equal(S_steps[:, j, :, 1:, :], S0.double().numpy()[:, :, 1:, :])


def test_one_token_is_a_decode_step():
    B, H_qk, H_v, d = 4, 2, 6, 16
    S0, (q, k, v, la, be) = _window(B, H_qk, H_v, d, 1, seed=24)
    o, S_steps = oracle.decode_multi(q, k, v, la, be, S0)
    o1, S1 = oracle.decode_step(q[:, 0], k[:, 0], v[:, 0], la[:, 0], be[:, 0], S0)
    np.testing.assert_array_equal(o[:, 0], o1)
    np.testing.assert_array_equal(S_steps[:, 0], S1)
