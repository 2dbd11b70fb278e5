"""Pins of the fp64 oracle against facts fixed by the state-update formula of
the bjdmk.com.cn article (section 2.1 "Gated DeltaNet 负责廉价压缩历史") and by
mathematics, independent of the oracle's own code.  CPU only.

Each ``pin_*`` takes an optional build of the C oracle, so that
``test_planted_mistakes_are_caught`` can run every pin against copies of the
oracle with a mistake planted in them (a flipped sign, a dropped decay, a
transposed state, a wrong head map, a pre-update readout, ...) and check
that each mistake fails at least one pin.
"""
import json
import os
import re
import shutil

import numpy as np
import pytest
import torch

import oracle
from linear_attention_12_b200 import inputs
from tests.chunk_form import chunked_prefill

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _case(T, H_qk, H_v, d, seed, dtype=torch.float32, s0=False, lens=None, alpha_mu=0.0):
    return inputs.make_prefill("t", lens or [T], H_qk, H_v, d=d, dtype=dtype, seed=seed,
                               s0=s0, alpha_mu=alpha_mu)


def _exact_unit_vectors(rng, n, d):
    """Unit vectors with exactly representable entries: 16 entries of +-1/4
    (4 entries of +-1/2 when d < 16) at random positions."""
    out = np.zeros((n, d), dtype=np.float32)
    m, val = (16, 0.25) if d >= 16 else (4, 0.5)
    for i in range(n):
        pos = rng.choice(d, size=m, replace=False)
        out[i, pos] = val * rng.choice([-1.0, 1.0], size=m)
    return out


# ---------------------------------------------------------------- pins
def pin_golden_hand_example_d2_L3(lib=None):
    """Hand-derived d=2, L=3 example (tests/golden/gdn_hand_d2_L3.json)."""
    g = json.load(open(os.path.join(GOLDEN, "gdn_hand_d2_L3.json")))
    q, k, v = (_f32(g[n])[:, None, :] for n in ("q", "k", "v"))
    la, be = _f32(g["log_alpha"])[:, None], _f32(g["beta"])[:, None]
    o, S = oracle.prefill(q, k, v, la, be, lib=lib)
    np.testing.assert_array_equal(o[:, 0, :], np.array(g["o"]))
    np.testing.assert_array_equal(S[0, 0], np.array(g["S_final"]))


def pin_decay_only_closed_form(lib=None):
    """beta = 0: S_t = alpha_t S_{t-1}, so S_L = exp(sum log alpha) S_0 and
    o_t = exp(g_t) S_0^T q_t."""
    c = _case(97, 2, 4, 16, seed=11, s0=True)
    be = torch.zeros_like(c.beta)
    o, S = oracle.prefill(c.q, c.k, c.v, c.log_alpha, be, S0=c.S0, lib=lib)
    g = np.cumsum(c.log_alpha.double().numpy(), axis=0)
    S0 = c.S0.double().numpy()
    for h in range(4):
        np.testing.assert_allclose(S[0, h], np.exp(g[-1, h]) * S0[0, h], rtol=1e-12, atol=0)
        qh = c.q[:, h // 2].double().numpy()
        ref = np.exp(g[:, h])[:, None] * (qh @ S0[0, h])
        np.testing.assert_allclose(o[:, h], ref, rtol=1e-11, atol=1e-300)


def pin_delta_write_exact_for_unit_keys(lib=None):
    """alpha = beta = 1 and ||k|| = 1 exactly: after the write S_t^T k_t = v_t,
    so reading with q_t = k_t returns v_t (from any S_0)."""
    rng = np.random.default_rng(5)
    T, d = 40, 128
    k = _exact_unit_vectors(rng, T, d)[:, None, :]
    v = _f32(rng.standard_normal((T, 1, d)))
    S0 = _f32(0.3 * rng.standard_normal((1, 1, d, d)))
    o, _ = oracle.prefill(k, k, v, np.zeros((T, 1), np.float32), np.ones((T, 1), np.float32),
                          S0=S0, lib=lib)
    np.testing.assert_allclose(o[:, 0], v[:, 0].astype(np.float64), rtol=0, atol=1e-13)


def pin_single_step_closed_form(lib=None):
    """L = 1: S_1 = alpha (I - beta k k^T) S_0 + beta k v^T, o_1 = S_1^T q."""
    rng = np.random.default_rng(7)
    d = 32
    q, k, v = (_f32(rng.standard_normal((1, 1, d))) for _ in range(3))
    S0 = _f32(rng.standard_normal((1, 1, d, d)))
    la, be = _f32([[-0.3]]), _f32([[0.7]])
    o, S = oracle.prefill(q, k, v, la, be, S0=S0, lib=lib)
    a, b = np.exp(np.float64(la[0, 0])), np.float64(be[0, 0])
    kk = k[0, 0].astype(np.float64)
    S1 = a * (np.eye(d) - b * np.outer(kk, kk)) @ S0[0, 0].astype(np.float64) \
        + b * np.outer(kk, v[0, 0].astype(np.float64))
    np.testing.assert_allclose(S[0, 0], S1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o[0, 0], S1.T @ q[0, 0].astype(np.float64), rtol=1e-12, atol=1e-13)


def pin_lookup_table_orthonormal_keys(lib=None):
    """alpha = beta = 1, k_t = e_t, S_0 = 0: S_t = sum_{j<=t} e_j v_j^T, so a
    query e_j returns v_j once token j was written and 0 before that (the
    associative-memory reading of the delta rule)."""
    d = T = 16
    rng = np.random.default_rng(3)
    k = np.eye(d, dtype=np.float32)[:T, None, :]
    v = _f32(rng.standard_normal((T, 1, 2 * d)))  # d_v != d_k catches a transposed state
    qidx = rng.integers(0, d, size=T)
    q = np.eye(d, dtype=np.float32)[qidx][:, None, :]
    o, S = oracle.prefill(q, k, v, np.zeros((T, 1), np.float32), np.ones((T, 1), np.float32),
                          lib=lib)
    for t in range(T):
        j = qidx[t]
        expect = v[j, 0].astype(np.float64) if j <= t else np.zeros(2 * d)
        np.testing.assert_array_equal(o[t, 0], expect)
    np.testing.assert_array_equal(S[0, 0], v[:, 0].astype(np.float64))


def pin_overwrite_replaces_not_adds(lib=None):
    """alpha = beta = 1, one unit key written twice with v then v': reading it
    returns v' (the delta rule replaces the stored value)."""
    d = 8
    k = np.zeros((2, 1, d), np.float32)
    k[:, 0, :4] = 0.5
    v = _f32([[[1, 2, 3, 4, 5, 6, 7, 8]], [[-1, 0, 2, 0, 1, 0, 3, 0]]])
    o, _ = oracle.prefill(k, k, v, np.zeros((2, 1), np.float32), np.ones((2, 1), np.float32),
                          lib=lib)
    np.testing.assert_array_equal(o[1, 0], v[1, 0].astype(np.float64))
    np.testing.assert_array_equal(o[0, 0], v[0, 0].astype(np.float64))


def pin_gqa_head_map_matches_replicated_heads(lib=None):
    """V head h reads QK head h // (H_v / H_qk): a GQA call equals the same
    call with q/k replicated to one QK head per V head."""
    c = _case(50, 2, 6, 16, seed=4, s0=True)
    o, S = oracle.prefill(c.q, c.k, c.v, c.log_alpha, c.beta, S0=c.S0, lib=lib)
    qr, kr = c.q.repeat_interleave(3, dim=1), c.k.repeat_interleave(3, dim=1)
    o2, S2 = oracle.prefill(qr, kr, c.v, c.log_alpha, c.beta, S0=c.S0)  # default build
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(S, S2)


def pin_literal_matrix_form(lib=None, d=8, T=300, lens=None):
    """The oracle equals the literal evaluation of the formula (explicit
    alpha (I - beta k k^T) matrices, numpy) to fp64 rounding."""
    c = _case(T, 2, 4, d, seed=d + T, s0=True, lens=lens)
    o, S = oracle.prefill(c.q, c.k, c.v, c.log_alpha, c.beta, S0=c.S0, cu_seqlens=c.cu_seqlens,
                          lib=lib)
    o2, S2 = oracle.literal_prefill(c.q, c.k, c.v, c.log_alpha, c.beta, S0=c.S0,
                                    cu_seqlens=c.cu_seqlens)
    assert np.abs(o - o2).max() <= 1e-13 * np.abs(o2).max()
    assert np.abs(S - S2).max() <= 1e-13 * np.abs(S2).max()


def pin_varlen_equals_separate_sequences(lib=None):
    c = _case(0, 2, 2, 16, seed=9, s0=True, lens=[17, 64, 1, 40])
    o, S = oracle.prefill(c.q, c.k, c.v, c.log_alpha, c.beta, S0=c.S0, cu_seqlens=c.cu_seqlens,
                          lib=lib)
    cu = c.cu_seqlens.tolist()
    for n in range(4):
        sl = slice(cu[n], cu[n + 1])
        on, Sn = oracle.prefill(c.q[sl], c.k[sl], c.v[sl], c.log_alpha[sl], c.beta[sl],
                                S0=c.S0[n:n + 1])
        np.testing.assert_array_equal(o[sl], on)
        np.testing.assert_array_equal(S[n], Sn[0])


PINS = [pin_golden_hand_example_d2_L3, pin_decay_only_closed_form,
        pin_delta_write_exact_for_unit_keys, pin_single_step_closed_form,
        pin_lookup_table_orthonormal_keys, pin_overwrite_replaces_not_adds,
        pin_gqa_head_map_matches_replicated_heads, pin_literal_matrix_form]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


@pytest.mark.parametrize("d,T,lens", [(128, 150, None), (16, 0, [5, 70, 33])])
def test_literal_matrix_form_more_shapes(d, T, lens):
    pin_literal_matrix_form(d=d, T=T, lens=lens)


def test_varlen_equals_separate_sequences():
    pin_varlen_equals_separate_sequences()


# ---------------------------------------------------------------- invariants
def test_nonexpansive_bound():
    """||k|| = 1, beta in [0,1], alpha in (0,1]: ||alpha (I - beta k k^T)||_2 <= alpha,
    hence ||S_t||_F <= alpha_t ||S_{t-1}||_F + beta_t ||v_t||."""
    c = _case(48, 1, 1, 32, seed=21, s0=True)
    T = c.T
    units = [(0, t, 0) for t in range(T + 1)]
    S0 = np.repeat(c.S0.double().numpy()[0, 0][None], T + 1, axis=0)
    S, _ = oracle.run_units(c.q, c.k, c.v, c.log_alpha, c.beta, units, S_init=S0, want_o=False)
    nrm = np.linalg.norm(S.reshape(T + 1, -1), axis=1)
    a = np.exp(c.log_alpha.double().numpy()[:, 0])
    b = c.beta.double().numpy()[:, 0]
    vn = np.linalg.norm(c.v.double().numpy()[:, 0], axis=1)
    assert np.all(nrm[1:] <= a * nrm[:-1] + b * vn + 1e-12)


def test_linear_in_v_and_S0():
    c = _case(70, 1, 3, 16, seed=8, s0=True)
    rng = np.random.default_rng(1)
    v2 = torch.from_numpy(_f32(rng.standard_normal(c.v.shape)))
    S02 = torch.from_numpy(_f32(rng.standard_normal(c.S0.shape)))
    a, b = 0.75, -1.5  # exact in fp32, and a*x + b*y of fp32 values is exact in fp64
    o1, S1 = oracle.prefill(c.q, c.k, c.v, c.log_alpha, c.beta, S0=c.S0)
    o2, S2 = oracle.prefill(c.q, c.k, v2, c.log_alpha, c.beta, S0=S02)
    v3 = (a * c.v.double() + b * v2.double()).float()
    S03 = (a * c.S0.double() + b * S02.double()).float()
    o3, S3 = oracle.prefill(c.q, c.k, v3, c.log_alpha, c.beta, S0=S03)
    # re-rounding the combined inputs to fp32 costs ~1e-7 relative
    np.testing.assert_allclose(o3, a * o1 + b * o2, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(S3, a * S1 + b * S2, rtol=1e-5, atol=1e-6)


def test_split_sequence_via_S0():
    """prefill(x[:m]) -> S_m, then prefill(x[m:], S0=S_m) equals prefill(x)."""
    c = _case(90, 1, 2, 16, seed=13)
    o, S = oracle.prefill(c.q, c.k, c.v, c.log_alpha, c.beta)
    m = 37
    oa, Sa = oracle.prefill(c.q[:m], c.k[:m], c.v[:m], c.log_alpha[:m], c.beta[:m])
    ob, Sb = oracle.prefill(c.q[m:], c.k[m:], c.v[m:], c.log_alpha[m:], c.beta[m:], S0=Sa)
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(Sb, S, rtol=0, atol=1e-14)


def test_bf16_inputs_widen_exactly():
    c = _case(30, 1, 3, 16, seed=2, dtype=torch.bfloat16)
    o, S = oracle.prefill(c.q, c.k, c.v, c.log_alpha, c.beta)
    o2, S2 = oracle.prefill(c.q.float(), c.k.float(), c.v.float(), c.log_alpha, c.beta)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(S, S2)


def test_decode_step_is_a_length_one_prefill():
    c = _case(3, 2, 4, 16, seed=31, s0=True, lens=[1, 1, 1])
    o, S = oracle.prefill(c.q, c.k, c.v, c.log_alpha, c.beta, S0=c.S0, cu_seqlens=c.cu_seqlens)
    o2, S2 = oracle.decode_step(c.q, c.k, c.v, c.log_alpha, c.beta, c.S0)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(S, S2)


def test_exact_rational_brute_force_d2():
    """d = 2, L = 3 with dyadic inputs and a nonzero S_0: exact rational
    evaluation of the literal formula (sympy) equals the oracle bit for bit."""
    sympy = pytest.importorskip("sympy")
    R = sympy.Rational
    k = [[R(1, 2), R(-3, 4)], [R(1), R(1, 4)], [R(-1, 2), R(1, 2)]]
    v = [[R(3), R(-1, 2)], [R(1, 8), R(2)], [R(-5, 4), R(1)]]
    q = [[R(1), R(1, 2)], [R(-1, 4), R(1)], [R(2), R(-1)]]
    beta = [R(1, 2), R(3, 4), R(1)]
    S0 = [[R(1, 4), R(0)], [R(-1, 2), R(1, 8)]]
    S = sympy.Matrix(S0)
    outs = []
    for t in range(3):
        kt = sympy.Matrix(k[t])
        S = (sympy.eye(2) - beta[t] * kt * kt.T) * S + beta[t] * kt * sympy.Matrix(v[t]).T
        outs.append([float(x) for x in (S.T * sympy.Matrix(q[t]))])
    f = lambda m: _f32(np.array(m, dtype=np.float64))
    o, Sf = oracle.prefill(f(q)[:, None, :], f(k)[:, None, :], f(v)[:, None, :],
                           np.zeros((3, 1), np.float32), f(beta)[:, None],
                           S0=f(S0)[None, None])
    np.testing.assert_array_equal(o[:, 0], np.array(outs))
    np.testing.assert_array_equal(Sf[0, 0], np.array(S.tolist(), dtype=np.float64))


@pytest.mark.parametrize("lens,C", [([200], 64), ([64], 64), ([1, 65, 129], 64), ([90], 16)])
def test_chunked_algebra_matches_oracle(lens, C):
    """The chunked (WY/UT) form the kernel implements reproduces the
    sequential oracle to fp64 rounding, partial chunks included."""
    c = _case(0, 2, 6, 32, seed=sum(lens), s0=True, lens=lens)
    o, S = oracle.prefill(c.q, c.k, c.v, c.log_alpha, c.beta, S0=c.S0, cu_seqlens=c.cu_seqlens)
    o2, S2 = chunked_prefill(c.q, c.k, c.v, c.log_alpha.numpy(), c.beta.numpy(),
                             S0=c.S0.numpy(), cu_seqlens=c.cu_seqlens.numpy(), C=C)
    assert np.abs(o - o2).max() <= 1e-12 * np.abs(o).max()
    assert np.abs(S - S2).max() <= 1e-12 * np.abs(S).max()


# ---------------------------------------------------------------- planted mistakes
# Each entry: (name, regex on gdn_oracle.c, replacement).  The regex must
# match exactly once, so an edit of the oracle that moves these lines makes
# this test fail loudly instead of silently testing nothing.
MUTANTS = [
    ("correction_sign", r"- alpha \* p\[j\]\)", "+ alpha * p[j])"),
    ("correction_without_alpha", r"- alpha \* p\[j\]\)", "- p[j])"),
    ("no_decay", r"Si\[j\] = alpha \* Si\[j\] \+ ki \* p\[j\]", "Si[j] = Si[j] + ki * p[j]"),
    ("beta_dropped", r"p\[j\] = beta \* \(", "p[j] = ("),
    # reads S^T instead of S (index kept in bounds for non-square states)
    ("transposed_prediction", r"p\[j\] \+= Si\[j\] \* ki;",
     "p[j] += S[(size_t)(j % dk) * dv + (i % dv)] * ki;"),
    ("head_map_modulo", r"const int hq = h / group;", "const int hq = h % J->H_qk;"),
    ("readout_uses_k", r"qbuf\[i\] = widen\(J->q,", "qbuf[i] = widen(J->k,"),
]


def _build_mutant(tmp_path, name, pattern, repl):
    src = open(oracle._SRC).read()
    new, n = re.subn(pattern, repl, src)
    assert n == 1, f"mutant {name}: pattern matched {n} times"
    p = tmp_path / f"mut_{name}.c"
    p.write_text(new)
    return oracle.build(force=True, src=str(p), out=str(tmp_path / f"libmut_{name}.so"))


@pytest.mark.parametrize("name,pattern,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistakes_are_caught(tmp_path, name, pattern, repl):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    lib = _build_mutant(tmp_path, name, pattern, repl)
    failed = []
    for pin in PINS:
        try:
            pin(lib=lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"planted mistake '{name}' passed every pin"
