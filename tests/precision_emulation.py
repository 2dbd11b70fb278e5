"""Where the prefill's error against the fp64 oracle comes from.

Not a test (pytest does not collect it): a CPU emulation of the chunked
prefill's rounding points, used to choose the 16-bit type of each tensor-core
operand.  The chunk algebra is the one the kernels use (the comment at the top
of ``gdn_prefill.cu``); every product is taken in fp32, and each operand
listed in a variant is rounded to its type before the product, as the
kernels' shared-memory tiles are.  Only the rounding points vary.

    python tests/precision_emulation.py [L]

prints the max-relative o error and the relative Frobenius S error of every
variant for three gate regimes (log_alpha = -softplus(N(mu, 1)), mu = 0, -2,
-6) on one QK head with three V heads.
"""
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import oracle  # noqa: E402
from linear_attention_12_b200 import inputs  # noqa: E402

C = 64
ROUND = {
    "bf16": lambda x: x.to(torch.bfloat16).float(),
    "fp16": lambda x: x.to(torch.float16).float(),
    "fp32": lambda x: x,
}

# variant: the type of each rounding point -- S (the state operand of K S and Q S),
# R (T_b and M o Q K^T, the record tiles), X, D (Delta in the output product),
# DD (d o Delta in the state update), O (the output)
VARIANTS = [
    ("all bf16", dict(S="bf16", R="bf16", X="bf16", D="bf16", DD="bf16", O="bf16")),
    ("S in fp32", dict(S="fp32", R="bf16", X="bf16", D="bf16", DD="bf16", O="bf16")),
    ("T_b, M o QK^T in fp32", dict(S="bf16", R="fp32", X="bf16", D="bf16", DD="bf16", O="bf16")),
    ("T_b, M o QK^T, X, Delta in fp16", dict(S="bf16", R="fp16", X="fp16", D="fp16", DD="bf16",
                                              O="bf16")),
    ("all intermediates fp32, o bf16", dict(S="fp32", R="fp32", X="fp32", D="fp32", DD="fp32",
                                            O="bf16")),
    ("everything fp32", dict(S="fp32", R="fp32", X="fp32", D="fp32", DD="fp32", O="fp32")),
]


def chunk_operators(K, Q, la, be):
    """T_b, M o Q K^T, gamma, d, gamma_C of one chunk (fp32)."""
    g = torch.cumsum(la, 0)
    M = torch.exp(g[:, None] - g[None, :]).tril()
    A = (be[:, None] * M * (K @ K.T)).tril(-1)
    T = torch.linalg.inv(torch.eye(C) + A)
    return T * be[None, :], M * (Q @ K.T), torch.exp(g), torch.exp(g[-1] - g), torch.exp(g[-1])


def run(case, h, v):
    r = {k: ROUND[t] for k, t in v.items()}
    hq = h // (case.H_v // case.H_qk)
    q, k = case.q[:, hq].float(), case.k[:, hq].float()
    vv, la, be = case.v[:, h].float(), case.log_alpha[:, h], case.beta[:, h]
    L = q.shape[0]
    S = torch.zeros(128, 128)
    o = torch.zeros(L, 128)
    for c0 in range(0, L, C):
        n = min(C, L - c0)
        K, Q, V = (torch.zeros(C, 128) for _ in range(3))
        K[:n], Q[:n], V[:n] = k[c0:c0 + n], q[c0:c0 + n], vv[c0:c0 + n]
        lac, bec = torch.zeros(C), torch.zeros(C)
        lac[:n], bec[:n] = la[c0:c0 + n], be[c0:c0 + n]
        Tb, MQ, gam, d, gC = chunk_operators(K, Q, lac, bec)
        d[n:] = 0
        Sr = r["S"](S)
        X = V - gam[:, None] * (K @ Sr)
        Dl = r["R"](Tb) @ r["X"](X)
        O = gam[:, None] * (Q @ Sr) + r["R"](MQ) @ r["D"](Dl)
        o[c0:c0 + n] = O[:n]
        S = gC * S + K.T @ r["DD"](Dl * d[:, None])
    return r["O"](o), S


def main():
    L = int(sys.argv[1]) if len(sys.argv) > 1 else 2048
    torch.set_grad_enabled(False)
    for mu in (0.0, -2.0, -6.0):
        case = inputs.make_prefill("emulation", [L], 1, 3, seed=5, alpha_mu=mu)
        o_ref, S_ref = oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, None,
                                      case.cu_seqlens)
        for name, v in VARIANTS:
            eo, es = [], []
            for h in range(3):
                o, S = run(case, h, v)
                ref = o_ref[:, h]
                eo.append(np.abs(o.double().numpy() - ref).max() / np.abs(ref).max())
                Sr = S_ref[0, h]
                es.append(np.linalg.norm(S.double().numpy() - Sr) / np.linalg.norm(Sr))
            print(f"mu={mu:5.1f}  {name:34s} o error {max(eo):.2e}  S error {max(es):.2e}")


if __name__ == "__main__":
    main()
