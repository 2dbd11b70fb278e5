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


def chunked_backward(q, k, v, log_alpha, beta, dO, S0=None, dS_final=None, cu_seqlens=None,
                     C=64):
    """Gradients of L = <dO, o> + <dS_final, S_final> in the chunk form the
    kernels use (T_b = T diag(beta), X = V - diag(gamma) K S, Delta = T_b X):
    a reverse pass over chunks carrying dS, the gradient of the state entering
    the chunk after it.  Per chunk, with dS' that gradient and S the entering
    state (d_r = exp(g_C - g_r), M the decay mask, QKm = M o Q K^T):

        dDelta = QKm^T dO + diag(d) K dS'          dX = T_b^T dDelta,  dV = dX
        dS     = gamma_C dS' + (diag(gamma) Q)^T dO - (diag(gamma) K)^T dX
        dQ     = diag(gamma) dO S^T + (M o dO Delta^T) K
        dK     = (M o dO Delta^T)^T Q - diag(gamma) dX S^T + diag(d) Delta dS'^T + (E + E^T) K
        with dT = dDelta X^T diag(beta), dA = strict_lower(-T^T dT T^T),
             E = dA o diag(beta) M (A's strict lower entries depend on k_r . k_j),
        dbeta_j = sum_r (dDelta X^T)_rj T_rj + sum_j' dA_jj' M_jj' (K K^T)_jj',

    and the gates through the cumulative log gates g (gamma, d, M, gamma_C
    are exponentials of g and of its differences), reverse-summed within the
    chunk into dlog_alpha.  Returns (dq, dk, dv, dlog_alpha, dbeta, dS0)."""
    qd, kd, vd = _widen(q), _widen(k), _widen(v)
    la = np.asarray(log_alpha, dtype=np.float64)
    be = np.asarray(beta, dtype=np.float64)
    dOd = np.asarray(dO, dtype=np.float64)
    T, H_qk, dk_ = qd.shape
    H_v, dv_ = vd.shape[1], vd.shape[2]
    grp = H_v // H_qk
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    dq, dk, dv = np.zeros_like(qd), np.zeros_like(kd), np.zeros_like(vd)
    dla, dbe = np.zeros_like(la), np.zeros_like(be)
    dS0 = np.zeros((N, H_v, dk_, dv_))
    for n in range(N):
        for h in range(H_v):
            hq = h // grp
            chunks = [(c0, min(cu[n + 1], c0 + C)) for c0 in range(cu[n], cu[n + 1], C)]
            # forward: the state entering every chunk
            S = np.zeros((dk_, dv_)) if S0 is None else np.asarray(S0[n, h], dtype=np.float64)
            entering = []
            for c0, c1 in chunks:
                entering.append(S)
                S = _chunk(qd, kd, vd, la, be, c0, c1, h, hq, S)["S_next"]
            dS = (np.zeros((dk_, dv_)) if dS_final is None
                  else np.asarray(dS_final[n, h], dtype=np.float64))
            for (c0, c1), S in reversed(list(zip(chunks, entering))):
                f = _chunk(qd, kd, vd, la, be, c0, c1, h, hq, S)
                K, Q, b, gam, dvec = f["K"], f["Q"], f["b"], f["gam"], f["dvec"]
                M, Tm, X, Delta, lows = f["M"], f["Tm"], f["X"], f["Delta"], f["lows"]
                Tb = Tm * b[None, :]
                dOc = dOd[c0:c1, h]
                KK, QK = K @ K.T, Q @ K.T
                dDelta = (M * QK).T @ dOc + dvec[:, None] * (K @ dS)
                dX = Tb.T @ dDelta
                dv[c0:c1, h] = dX
                MdOD = M * (dOc @ Delta.T)
                dq[c0:c1, hq] += gam[:, None] * (dOc @ S.T) + MdOD @ K
                dTb = dDelta @ X.T
                dTm = dTb * b[None, :]
                dA = lows * (-Tm.T @ dTm @ Tm.T)
                E = dA * b[:, None] * M
                dk[c0:c1, hq] += (MdOD.T @ Q - gam[:, None] * (dX @ S.T)
                                  + dvec[:, None] * (Delta @ dS.T) + (E + E.T) @ K)
                dbe[c0:c1, h] = np.sum(dTb * Tm, axis=0) + np.sum(dA * M * KK, axis=1)
                # the gates, through g
                dg = gam * (np.sum(dOc * (Q @ S), axis=1) - np.sum(dX * (K @ S), axis=1))
                dM = (dOc @ Delta.T) * QK + dA * b[:, None] * KK  # dL/dM (M not included)
                dg += np.sum(dM * M, axis=1) - np.sum(dM * M, axis=0)
                ddv = np.sum((K @ dS) * Delta, axis=1) * dvec
                dg -= ddv
                dg[-1] += ddv.sum() + gam[-1] * np.sum(dS * S)
                dla[c0:c1, h] = np.cumsum(dg[::-1])[::-1]
                dS = gam[-1] * dS + (gam[:, None] * Q).T @ dOc - (gam[:, None] * K).T @ dX
            dS0[n, h] = dS
    return dq, dk, dv, dla, dbe, dS0


def _chunk(qd, kd, vd, la, be, c0, c1, h, hq, S):
    """Forward quantities of one chunk in the kernels' form."""
    K, Q, V = kd[c0:c1, hq], qd[c0:c1, hq], vd[c0:c1, h]
    b = be[c0:c1, h]
    g = np.cumsum(la[c0:c1, h])
    gam = np.exp(g)
    L = c1 - c0
    lows = np.tril(np.ones((L, L)), -1)
    M = np.exp(np.where(np.tril(np.ones((L, L))) > 0, g[:, None] - g[None, :], -np.inf))
    A = lows * b[:, None] * M * (K @ K.T)
    Tm = np.linalg.inv(np.eye(L) + A)
    X = V - gam[:, None] * (K @ S)
    Delta = (Tm * b[None, :]) @ X
    dvec = np.exp(g[-1] - g)
    return dict(K=K, Q=Q, b=b, gam=gam, dvec=dvec, M=M, Tm=Tm, X=X, Delta=Delta, lows=lows,
                S_next=gam[-1] * S + (dvec[:, None] * K).T @ Delta)
