"""Test-only numpy fp64 evaluation of the GDN recurrence in chunked (WY/UT) form.

The bjdmk.com.cn article (section 2.1) says the recurrence is made
chunk-parallel with the WY representation but prints no formulas.  The form
below is re-derived from the state-update formula alone:

within a chunk with entry state S_0 and cumulative log-gates g_r = sum_{i<=r}
log alpha_i (gamma_r = exp g_r), unrolling the recurrence gives

    S_r = gamma_r S_0 + sum_{j<=r} exp(g_r - g_j) k_j u_j^T,
    u_r = beta_r (v_r - alpha_r S_{r-1}^T k_r),

so the write vectors U = [u_r] solve the unit-lower-triangular system

    (I + A) U = diag(beta) V - diag(beta gamma) K S_0,
    A_rj = beta_r exp(g_r - g_j) (k_r . k_j)   for j < r, else 0.

With T = (I + A)^{-1}, W = T diag(beta gamma) K and U0 = T diag(beta) V:

    Delta     = U0 - W S_0                      (the true write vectors)
    O         = diag(gamma) Q S_0 + (M * Q K^T) Delta,  M_rj = exp(g_r - g_j), j <= r
    S_next    = gamma_C S_0 + Ktil^T Delta,     Ktil_j = exp(g_C - g_j) k_j.

This module is neither the oracle nor the CUDA path; the tests check it
against the oracle, which makes it a statement of the algebra the kernel uses.
"""
import numpy as np


def _widen(a):
    import oracle
    return oracle._widen(a)


def chunked_prefill(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, C=64):
    qd, kd, vd = _widen(q), _widen(k), _widen(v)
    la = np.asarray(log_alpha, dtype=np.float64)
    be = np.asarray(beta, dtype=np.float64)
    T, H_qk, dk = qd.shape
    H_v, dv = vd.shape[1], vd.shape[2]
    grp = H_v // H_qk
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    o = np.zeros((T, H_v, dv))
    S_fin = np.zeros((N, H_v, dk, dv))
    for n in range(N):
        for h in range(H_v):
            S = np.zeros((dk, dv)) if S0 is None else np.asarray(S0[n, h], dtype=np.float64)
            for c0 in range(cu[n], cu[n + 1], C):
                c1 = min(cu[n + 1], c0 + C)
                K, Q, V = kd[c0:c1, h // grp], qd[c0:c1, h // grp], vd[c0:c1, h]
                b = be[c0:c1, h]
                g = np.cumsum(la[c0:c1, h])
                gam = np.exp(g)
                L = c1 - c0
                diff = g[:, None] - g[None, :]
                low_strict = np.tril(np.ones((L, L)), -1)
                low_incl = np.tril(np.ones((L, L)))
                decay = np.exp(np.where(low_incl > 0, diff, -np.inf))
                A = low_strict * b[:, None] * decay * (K @ K.T)
                Tm = np.linalg.inv(np.eye(L) + A)
                W = Tm @ ((b * gam)[:, None] * K)
                U0 = Tm @ (b[:, None] * V)
                Delta = U0 - W @ S
                o[c0:c1, h] = gam[:, None] * (Q @ S) + (decay * (Q @ K.T)) @ Delta
                Ktil = np.exp(g[-1] - g)[:, None] * K
                S = gam[-1] * S + Ktil.T @ Delta
            S_fin[n, h] = S
    return o, S_fin
