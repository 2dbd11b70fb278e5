"""Seeded synthetic inputs for the GDN layer: the only code shared by the CUDA
path's tests/benchmark and the CPU oracle.  It holds none of the method's
arithmetic -- only the input distributions.

Recipe (shapes and distributions of the workloads described for the GDN layer
of Qwen3.8-Flash-Next: 16 QK heads shared by 48 V heads, head dim 128):

* one ``torch.Generator`` (CPU) seeded with ``seed``; tensors drawn in the
  order q, k, v, log_alpha, beta, S0, each in token blocks of ``BLOCK`` rows;
* q, k ~ N(0, 1) in fp32, L2-normalised per (token, head) in fp32, then cast
  to the I/O dtype (bf16 or fp32);
* v ~ N(0, 1), cast to the I/O dtype;
* log_alpha = -softplus(N(mu, 1)) with mu = 0 (mu = -2 for long-memory
  gates), beta = sigmoid(N(0, 1)); both fp32, one scalar per (token, V head);
* S0 = 0.02 * N(0, 1), fp32, or absent (zeros);
* packed variable-length batches draw their lengths first, uniformly in
  [lo, hi], from the same generator; cu_seqlens is their prefix sum.

Front-end inputs (the raw projections before the short convolution): q_raw,
k_raw, v_raw ~ N(0, 1) in the I/O dtype, gate pre-activations a, b ~ N(0, 1)
fp32, convolution weights 0.5 * N(0, 1) fp32 ``[(2 H_qk + H_v) d, 4]``; drawn in
the order q_raw, k_raw, v_raw, a, b, conv_w.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.nn.functional as F

BLOCK = 4096


@dataclasses.dataclass
class PrefillCase:
    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    log_alpha: torch.Tensor
    beta: torch.Tensor
    S0: torch.Tensor | None
    cu_seqlens: torch.Tensor
    H_qk: int
    H_v: int
    d: int

    @property
    def T(self) -> int:
        return self.q.shape[0]

    @property
    def N(self) -> int:
        return self.cu_seqlens.numel() - 1


def _normal(gen, shape, mu=0.0):
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    return x + mu if mu else x


def _draw_rows(gen, T, row_shape, dtype, unit_norm):
    out = torch.empty((T, *row_shape), dtype=dtype)
    for t0 in range(0, T, BLOCK):
        t1 = min(T, t0 + BLOCK)
        x = _normal(gen, (t1 - t0, *row_shape))
        if unit_norm:
            x = x / x.norm(dim=-1, keepdim=True)
        out[t0:t1] = x.to(dtype)
    return out


def _draw_gates(gen, T, H_v, mu):
    la = torch.empty((T, H_v), dtype=torch.float32)
    for t0 in range(0, T, BLOCK):
        t1 = min(T, t0 + BLOCK)
        la[t0:t1] = -F.softplus(_normal(gen, (t1 - t0, H_v), mu))
    be = torch.empty((T, H_v), dtype=torch.float32)
    for t0 in range(0, T, BLOCK):
        t1 = min(T, t0 + BLOCK)
        be[t0:t1] = torch.sigmoid(_normal(gen, (t1 - t0, H_v)))
    return la, be


def make_prefill(name, seqlens, H_qk, H_v, d=128, dtype=torch.bfloat16, seed=0,
                 s0=False, alpha_mu=0.0, varlen_range=None) -> PrefillCase:
    """Draw one prefill case.  ``seqlens`` is a list of lengths, or None with
    ``varlen_range=(n, lo, hi)`` to draw n lengths uniformly in [lo, hi]."""
    gen = torch.Generator().manual_seed(seed)
    if varlen_range is not None:
        n, lo, hi = varlen_range
        seqlens = torch.randint(lo, hi + 1, (n,), generator=gen).tolist()
    cu = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    T = int(cu[-1])
    q = _draw_rows(gen, T, (H_qk, d), dtype, True)
    k = _draw_rows(gen, T, (H_qk, d), dtype, True)
    v = _draw_rows(gen, T, (H_v, d), dtype, False)
    la, be = _draw_gates(gen, T, H_v, alpha_mu)
    S0 = None
    if s0:
        S0 = 0.02 * _normal(gen, (len(seqlens), H_v, d, d))
    return PrefillCase(name, q, k, v, la, be, S0, cu, H_qk, H_v, d)


# The five workloads, by what they are.  The tiny one is small enough for the
# oracle to finish in well under a second.
def tiny_fp32():
    """B=1, L=256, 1 QK head, 1 V head, d=128, all fp32, S0 = 0, seed 0."""
    return make_prefill("tiny_fp32_L256", [256], 1, 1, dtype=torch.float32, seed=0)


def qwen_prefill_32k(L=32768):
    """B=1, L=32768, 16 QK / 48 V heads, d=128, bf16 q/k/v, fp32 gates, S0 = 0."""
    return make_prefill(f"prefill_L{L}_h16x48", [L], 16, 48, seed=1)


def varlen_8seq():
    """8 packed sequences, lengths uniform in [1024, 8192], S0 ~ N(0, 0.02^2)."""
    return make_prefill("varlen_8seq_1k_8k", None, 16, 48, seed=2, s0=True,
                        varlen_range=(8, 1024, 8192))


def long_256k(L=262144):
    """B=1, L=262144, long-memory gates log_alpha = -softplus(N(-2, 1))."""
    return make_prefill(f"prefill_L{L}_longmem", [L], 16, 48, seed=3, alpha_mu=-2.0)


@dataclasses.dataclass
class DecodeCase:
    B: int
    H_qk: int
    H_v: int
    d: int
    S0: torch.Tensor  # [B, H_v, d, d] fp32
    seed: int

    def step(self, s: int, dtype=torch.bfloat16):
        """Inputs of decode step ``s``: a generator seeded ``seed * 10**6 + s``."""
        gen = torch.Generator().manual_seed(self.seed * 10**6 + s)
        q = _draw_rows(gen, self.B, (self.H_qk, self.d), dtype, True)
        k = _draw_rows(gen, self.B, (self.H_qk, self.d), dtype, True)
        v = _draw_rows(gen, self.B, (self.H_v, self.d), dtype, False)
        la, be = _draw_gates(gen, self.B, self.H_v, 0.0)
        return q, k, v, la, be

    def window(self, s: int, M: int, dtype=torch.bfloat16):
        """Inputs of steps ``s .. s+M-1`` stacked on a token axis (a verify window
        of M drafted tokens): q, k ``[B, M, H_qk, d]``, v ``[B, M, H_v, d]``,
        gates ``[B, M, H_v]`` -- the same values ``step`` draws one by one."""
        steps = [self.step(s + j, dtype) for j in range(M)]
        return tuple(torch.stack([st[i] for st in steps], dim=1) for i in range(5))


def make_decode(B=256, H_qk=16, H_v=48, d=128, seed=4) -> DecodeCase:
    """Batched decode: B sequences, persistent fp32 states from 0.02 * N(0, 1)."""
    gen = torch.Generator().manual_seed(seed)
    S0 = torch.empty((B, H_v, d, d), dtype=torch.float32)
    for b0 in range(0, B, 16):
        b1 = min(B, b0 + 16)
        S0[b0:b1] = 0.02 * _normal(gen, (b1 - b0, H_v, d, d))
    return DecodeCase(B, H_qk, H_v, d, S0, seed)


def batched_decode_256():
    """256 sequences x 48 V heads (16 QK heads), d=128, 512 steps from seed 4."""
    return make_decode(256, 16, 48, 128, seed=4)


@dataclasses.dataclass
class FrontendCase:
    name: str
    q_raw: torch.Tensor
    k_raw: torch.Tensor
    v_raw: torch.Tensor
    a: torch.Tensor
    b: torch.Tensor
    conv_w: torch.Tensor
    cu_seqlens: torch.Tensor
    H_qk: int
    H_v: int
    d: int

    @property
    def T(self) -> int:
        return self.q_raw.shape[0]


def make_frontend(name, seqlens, H_qk, H_v, d=128, dtype=torch.bfloat16, seed=0) -> FrontendCase:
    """Draw the raw inputs of the front end for packed sequences of ``seqlens``."""
    gen = torch.Generator().manual_seed(seed)
    cu = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    T = int(cu[-1])
    q = _draw_rows(gen, T, (H_qk, d), dtype, False)
    k = _draw_rows(gen, T, (H_qk, d), dtype, False)
    v = _draw_rows(gen, T, (H_v, d), dtype, False)
    a = _draw_rows(gen, T, (H_v,), torch.float32, False)
    b = _draw_rows(gen, T, (H_v,), torch.float32, False)
    w = 0.5 * _normal(gen, ((2 * H_qk + H_v) * d, 4))
    return FrontendCase(name, q, k, v, a, b, w, cu, H_qk, H_v, d)
