"""Pins of the front-end oracle (oracle/frontend.py) to facts outside itself:
the identity and impulse responses of a width-4 causal convolution, the
independence of packed sequences, the decode-step ring state against the
prefill form, the closed forms of the gate activations, SiLU and the L2
normalisation.  CPU only."""
import numpy as np
import pytest

from oracle import frontend as fe

D = 8  # small head dim for the pins (the front end is per channel / per head)


def _raw(rng, T, H_qk, H_v, d=D):
    return (rng.standard_normal((T, H_qk, d)), rng.standard_normal((T, H_qk, d)),
            rng.standard_normal((T, H_v, d)), rng.standard_normal((T, H_v)),
            rng.standard_normal((T, H_v)))


def test_identity_kernel_passes_inputs_through():
    rng = np.random.default_rng(0)
    q, k, v, a, b = _raw(rng, 9, 1, 2)
    w = np.zeros(((2 + 2) * D, 4))
    w[:, 3] = 1.0  # only the current token
    oq, ok, ov, _, _ = fe.frontend(q, k, v, w, a, b, eps=0.0)
    np.testing.assert_allclose(ov, v, rtol=0, atol=0)
    np.testing.assert_allclose(oq, q / np.linalg.norm(q, axis=-1, keepdims=True), rtol=1e-14)
    np.testing.assert_allclose(ok, k / np.linalg.norm(k, axis=-1, keepdims=True), rtol=1e-14)


def test_impulse_response_reads_the_taps_in_time_order():
    # one nonzero input token t0 in a sequence; y[t0 + j] = w[:, 3 - j] * x[t0] for j = 0..3
    T, t0 = 12, 4
    v = np.zeros((T, 1, D))
    e = np.arange(1, D + 1, dtype=np.float64)
    v[t0, 0] = e
    q = np.zeros((T, 1, D))
    w = np.zeros((3 * D, 4))
    taps = np.array([0.5, -2.0, 3.0, 7.0])
    w[2 * D:] = taps
    _, _, ov, _, _ = fe.frontend(q, q, v, w, np.zeros((T, 1)), np.zeros((T, 1)))
    for t in range(T):
        j = t - t0
        want = taps[3 - j] * e if 0 <= j <= 3 else np.zeros(D)
        np.testing.assert_array_equal(ov[t, 0], want)


def test_history_does_not_cross_sequence_boundaries():
    rng = np.random.default_rng(1)
    q, k, v, a, b = _raw(rng, 17, 2, 4)
    w = rng.standard_normal(((4 + 4) * D, 4))
    cu = [0, 5, 5, 12, 17]
    packed = fe.frontend(q, k, v, w, a, b, cu_seqlens=cu, act="silu")
    for n in range(4):
        s0, s1 = cu[n], cu[n + 1]
        if s1 == s0:
            continue
        one = fe.frontend(q[s0:s1], k[s0:s1], v[s0:s1], w, a[s0:s1], b[s0:s1], act="silu")
        for x, y in zip(packed, one):
            np.testing.assert_allclose(x[s0:s1], y, rtol=1e-14, atol=1e-14)


def test_decode_steps_equal_the_prefill_form():
    rng = np.random.default_rng(2)
    T, H_qk, H_v = 7, 2, 6
    q, k, v, a, b = _raw(rng, T, H_qk, H_v)
    w = rng.standard_normal(((2 * H_qk + H_v) * D, 4))
    ref = fe.frontend(q, k, v, w, a, b, act="silu")
    state = np.zeros((1, 3, (2 * H_qk + H_v) * D))
    for t in range(T):
        out = fe.frontend_decode_step(q[t:t + 1], k[t:t + 1], v[t:t + 1], w, a[t:t + 1],
                                      b[t:t + 1], state, act="silu")
        state = out[5]
        for x, y in zip(out[:5], ref):
            np.testing.assert_allclose(x[0], y[t], rtol=1e-13, atol=1e-14)


def test_gate_activations_closed_forms():
    a = np.array([0.0, 50.0, -50.0, 1.0])
    la = -fe.softplus(a)
    assert la[0] == pytest.approx(-np.log(2.0), rel=1e-15)
    assert la[1] == pytest.approx(-50.0, rel=1e-15)  # softplus(a) -> a for large a
    assert la[2] == pytest.approx(-np.exp(-50.0), rel=1e-12)  # -> e^a for very negative a
    assert la[3] == pytest.approx(-np.log1p(np.e), rel=1e-15)
    bt = fe.sigmoid(np.array([0.0, 2.0]))
    assert bt[0] == 0.5
    assert bt[1] == pytest.approx(np.exp(2.0) / (1.0 + np.exp(2.0)), rel=1e-15)


def test_silu_and_l2_norm():
    y = np.array([[0.0, 1.0, -1.0, 30.0]])
    s = fe._act(y, "silu")
    np.testing.assert_allclose(s, [[0.0, 1 / (1 + np.exp(-1)), -1 / (1 + np.e), 30.0]],
                               rtol=1e-13)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, D)) * 3.0
    n = fe._l2norm(x, 0.0)
    np.testing.assert_allclose(np.linalg.norm(n, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(fe._l2norm(7.0 * x, 0.0), n, rtol=1e-14)  # scale invariance


def test_sampled_rows_equal_full_computation():
    rng = np.random.default_rng(4)
    q, k, v, a, b = _raw(rng, 30, 1, 3)
    w = rng.standard_normal((5 * D, 4))
    cu = [0, 11, 30]
    full = fe.frontend(q, k, v, w, a, b, cu_seqlens=cu)
    rows = [0, 3, 10, 11, 12, 14, 29]
    part = fe.frontend(q, k, v, w, a, b, cu_seqlens=cu, rows=rows)
    for x, y in zip(part, full):
        np.testing.assert_allclose(x, y[rows], rtol=1e-15, atol=0)
