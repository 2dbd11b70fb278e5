"""Pins of the backward oracle (oracle/backward.py): every gradient against
central finite differences of a loss computed with the explicit-matrix
evaluation of the state-update formula (oracle.literal_prefill, numpy,
independent of the backward code), on tiny packed inputs in fp64; plus the
closed forms of two special cases.  CPU only."""
import numpy as np
import pytest

import oracle
from oracle import backward

D = 4


def _case(seed, lens=(3, 4), H_qk=1, H_v=2, with_s0=True):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N = len(lens)
    x = dict(q=rng.standard_normal((T, H_qk, D)), k=rng.standard_normal((T, H_qk, D)),
             v=rng.standard_normal((T, H_v, D)),
             log_alpha=-np.log1p(np.exp(rng.standard_normal((T, H_v)))),
             beta=1 / (1 + np.exp(-rng.standard_normal((T, H_v)))),
             S0=0.3 * rng.standard_normal((N, H_v, D, D)) if with_s0 else np.zeros((N, H_v, D, D)))
    x["k"] /= np.linalg.norm(x["k"], axis=-1, keepdims=True)
    dO = rng.standard_normal((T, H_v, D))
    dSf = rng.standard_normal((N, H_v, D, D))
    return x, cu, dO, dSf


def _loss(x, cu, dO, dSf):
    o, S = oracle.literal_prefill(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S0=x["S0"],
                                  cu_seqlens=cu)
    return float(np.sum(o * dO) + np.sum(S * dSf))


def _fd(x, cu, dO, dSf, name, eps=1e-6):
    g = np.zeros_like(x[name])
    for idx in np.ndindex(*x[name].shape):
        xp = {k2: v2.copy() for k2, v2 in x.items()}
        xm = {k2: v2.copy() for k2, v2 in x.items()}
        xp[name][idx] += eps
        xm[name][idx] -= eps
        g[idx] = (_loss(xp, cu, dO, dSf) - _loss(xm, cu, dO, dSf)) / (2 * eps)
    return g


@pytest.mark.parametrize("seed", [0, 1])
def test_every_gradient_matches_finite_differences(seed):
    x, cu, dO, dSf = _case(seed)
    got = backward.prefill_backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dO,
                                    S0=x["S0"], dS_final=dSf, cu_seqlens=cu)
    for name, g in zip(["q", "k", "v", "log_alpha", "beta", "S0"], got):
        fd = _fd(x, cu, dO, dSf, name)
        np.testing.assert_allclose(g, fd, rtol=1e-6, atol=1e-7, err_msg=name)


def test_without_initial_state_or_state_gradient():
    # S0 = 0 and no gradient through the final state: only the outputs matter
    x, cu, dO, _ = _case(2, lens=(5,), H_qk=2, H_v=2, with_s0=False)
    dSf = np.zeros((1, 2, D, D))
    got = backward.prefill_backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dO,
                                    cu_seqlens=cu)
    for name, g in zip(["q", "k", "v", "log_alpha", "beta"], got[:5]):
        np.testing.assert_allclose(g, _fd(x, cu, dO, dSf, name), rtol=1e-6, atol=1e-7,
                                   err_msg=name)


def test_pure_decay_closed_form():
    # beta = 0: S_t = exp(g_t) S0 with g_t the cumulative log gate, o_t = S_t^T q_t, so
    # dS0 = sum_t exp(g_t) q_t do_t^T + exp(g_T) dS_final and dv = 0
    x, cu, dO, dSf = _case(3, lens=(6,), H_qk=1, H_v=1)
    x["beta"][:] = 0.0
    dq, dk, dv, dla, dbe, dS0 = backward.prefill_backward(
        x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dO, S0=x["S0"], dS_final=dSf,
        cu_seqlens=cu)
    g = np.cumsum(x["log_alpha"][:, 0])
    want = sum(np.exp(g[t]) * np.outer(x["q"][t, 0], dO[t, 0]) for t in range(6))
    want = want + np.exp(g[-1]) * dSf[0, 0]
    np.testing.assert_allclose(dS0[0, 0], want, rtol=1e-12)
    np.testing.assert_array_equal(dv, 0.0)
    np.testing.assert_allclose(dk, 0.0, atol=1e-15)  # k only enters through beta k k^T and beta k v^T


@pytest.mark.parametrize("C,lens,H_qk,H_v", [(4, (13, 0, 9), 1, 2), (8, (17,), 2, 4),
                                              (16, (5, 40), 1, 3)])
def test_chunk_form_of_the_gradients_equals_the_oracle(C, lens, H_qk, H_v):
    # the chunked backward the kernels follow (tests/chunk_form.py) against the
    # token-by-token reverse mode, on ragged and empty sequences with grouped heads
    from tests.chunk_form import chunked_backward
    rng = np.random.default_rng(C)
    T, N, d = sum(lens), len(lens), 8
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    q = rng.standard_normal((T, H_qk, d))
    k = rng.standard_normal((T, H_qk, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H_v, d))
    la = -np.log1p(np.exp(rng.standard_normal((T, H_v))))
    be = 1 / (1 + np.exp(-rng.standard_normal((T, H_v))))
    S0 = 0.3 * rng.standard_normal((N, H_v, d, d))
    dO = rng.standard_normal((T, H_v, d))
    dSf = rng.standard_normal((N, H_v, d, d))
    ref = backward.prefill_backward(q, k, v, la, be, dO, S0=S0, dS_final=dSf, cu_seqlens=cu)
    got = chunked_backward(q, k, v, la, be, dO, S0=S0, dS_final=dSf, cu_seqlens=cu, C=C)
    for name, a, b in zip(["dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"], got, ref):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12, err_msg=name)
