"""fp64 CPU oracle of the GDN prefill's gradients -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` may import this module; it shares no code with the CUDA
library.

The forward pass is the state-update formula of the bjdmk.com.cn article
"为什么 Qwen3.8-Flash-Next 值得单独跑一遍", section 2.1, with readout
``o_t = S_t^T q_t``.  Written in the expanded form of the same section (the
new value minus what the memory already predicts),

    p_t = S_{t-1}^T k_t                  (the memory's prediction of v_t)
    w_t = beta_t (v_t - alpha_t p_t)     (the write vector)
    S_t = alpha_t S_{t-1} + k_t w_t^T,   o_t = S_t^T q_t,

its reverse mode, token by token from the last one, is (G = dL/dS_t):

    G      += q_t do_t^T                  dq_t += S_t do_t
    dw      = G^T k_t
    dk_t   += G w_t - alpha_t beta_t S_{t-1} dw
    dv_t    = beta_t dw
    dbeta_t = dw . (v_t - alpha_t p_t)
    dalpha  = <G, S_{t-1}> - beta_t dw . p_t,   dlog_alpha_t = alpha_t dalpha
    G      <- alpha_t G - alpha_t beta_t k_t dw^T

and dS0 is G after the first token.  Query/key heads shared by several value
heads (grouped layout) sum the gradients of their value heads.  The pages
print no backward pass; this is the chain rule of the forward formula.
Plain loops over tokens, for small sizes.
"""
from __future__ import annotations

import numpy as np

from . import _widen


def prefill_backward(q, k, v, log_alpha, beta, dO, S0=None, dS_final=None, cu_seqlens=None):
    """Gradients of ``L = <dO, o> + <dS_final, S_final>`` for the prefill over
    packed sequences.  Inputs in the library's layouts (q, k ``[T, H_qk, d]``,
    v and dO ``[T, H_v, d]``, gates ``[T, H_v]``, states ``[N, H_v, d, d]``).
    Returns ``(dq, dk, dv, dlog_alpha, dbeta, dS0)`` in fp64."""
    qd, kd, vd = _widen(q), _widen(k), _widen(v)
    la, be, dOd = _widen(log_alpha), _widen(beta), _widen(dO)
    T, H_qk, dk_ = qd.shape
    H_v, dv_ = vd.shape[1], vd.shape[2]
    grp = H_v // H_qk
    cu = [0, T] if cu_seqlens is None else [int(c) for c in np.asarray(cu_seqlens).ravel()]
    N = len(cu) - 1
    S0d = np.zeros((N, H_v, dk_, dv_)) if S0 is None else _widen(S0)
    dSf = np.zeros((N, H_v, dk_, dv_)) if dS_final is None else _widen(dS_final)
    dq, dk = np.zeros_like(qd), np.zeros_like(kd)
    dv, dla, dbe = np.zeros_like(vd), np.zeros_like(la), np.zeros_like(be)
    dS0 = np.zeros_like(S0d)
    for n in range(N):
        t0, t1 = cu[n], cu[n + 1]
        for h in range(H_v):
            hq = h // grp
            # forward, keeping every state
            states = [S0d[n, h].copy()]
            for t in range(t0, t1):
                S = states[-1]
                a, b = np.exp(la[t, h]), be[t, h]
                kt, vt = kd[t, hq], vd[t, h]
                w = b * (vt - a * (S.T @ kt))
                states.append(a * S + np.outer(kt, w))
            # reverse
            G = dSf[n, h].copy()
            for t in range(t1 - 1, t0 - 1, -1):
                S_prev, S_t = states[t - t0], states[t - t0 + 1]
                a, b = np.exp(la[t, h]), be[t, h]
                kt, vt, qt, dot = kd[t, hq], vd[t, h], qd[t, hq], dOd[t, h]
                G = G + np.outer(qt, dot)
                dq[t, hq] += S_t @ dot
                p = S_prev.T @ kt
                w = b * (vt - a * p)
                dw = G.T @ kt
                dk[t, hq] += G @ w - a * b * (S_prev @ dw)
                dv[t, h] = b * dw
                dbe[t, h] = dw @ (vt - a * p)
                dla[t, h] = a * (np.sum(G * S_prev) - b * (dw @ p))
                G = a * G - a * b * np.outer(kt, dw)
            dS0[n, h] = G
    return dq, dk, dv, dla, dbe, dS0
