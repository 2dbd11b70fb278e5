"""fp64 CPU oracle for the GDN front end -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` (and the oracle's own callers listed in ``oracle/__init__.py``)
may import this module; it shares no code with the CUDA library.

The front end is the step that turns a layer's raw projections into the
recurrence's inputs.  What the pages fix and what is read into them:

* Short convolution -- jianying88.com article "Qwen3.8-Flash-Next混合注意力
  深度解析…", section 三 (config ``linear_conv_kernel_dim: 4``: the GDN layer
  stacks a short convolution of kernel width 4 to capture local detail).  The
  pages print no formula; the plain reading is a causal depthwise convolution
  of every q, k and v channel within its sequence,

      y[t, c] = sum_{i=0..3} w[c, i] * x[t - 3 + i, c],   x = 0 before the sequence start,

  so tap 3 weighs the current token.
* Activation after the convolution -- the pages name none.  ``act = "none"``
  is the plain reading; ``act = "silu"`` (y * sigmoid(y)) is offered as well.
* q, k L2-normalised per (token, head), and the gates
  ``log_alpha = -softplus(a)``, ``beta = sigmoid(b)`` -- the recipes of the
  workloads the layer is measured on (q and k L2-normalised per token; the
  forget gate's log as minus softplus of a normal draw; beta as its sigmoid).
  The normalisation divides by ``sqrt(sum x^2 + eps)`` (``eps`` a reading).

Channel layout of the convolution weight: ``[(2 H_qk + H_v) d, 4]``, the q
channels (head-major), then k, then v.  The decode-step form keeps, per
sequence, the last three raw input rows ``[B, 3, (2 H_qk + H_v) d]`` (oldest
first).
"""
from __future__ import annotations

import numpy as np

from . import _as_np, _widen


def _act(y: np.ndarray, act: str) -> np.ndarray:
    if act == "none":
        return y
    if act == "silu":
        return y / (1.0 + np.exp(-y))
    raise ValueError(act)


def _l2norm(x: np.ndarray, eps: float) -> np.ndarray:
    """Per-row L2 normalisation over the last axis."""
    return x / np.sqrt((x * x).sum(axis=-1, keepdims=True) + eps)


def softplus(a: np.ndarray) -> np.ndarray:
    """log(1 + e^a), evaluated without overflow."""
    return np.logaddexp(0.0, a)


def sigmoid(b: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-b))


def causal_conv(x: np.ndarray, w: np.ndarray, cu_seqlens) -> np.ndarray:
    """Width-4 causal depthwise convolution of ``x [T, C]`` with ``w [C, 4]``,
    restarted at every sequence start; a direct sum over the taps."""
    cu = [int(c) for c in cu_seqlens]
    y = np.zeros_like(x)
    for n in range(len(cu) - 1):
        t0, t1 = cu[n], cu[n + 1]
        for t in range(t0, t1):
            acc = np.zeros(x.shape[1])
            for i in range(4):
                tt = t - 3 + i
                if tt >= t0:
                    acc = acc + w[:, i] * x[tt]
            y[t] = acc
    return y


def frontend(q_raw, k_raw, v_raw, conv_w, a, b, cu_seqlens=None, act="none", eps=1e-6,
             rows=None):
    """Front end of a prefill.  Returns ``(q, k, v, log_alpha, beta)`` in fp64
    with the shapes of the inputs.

    ``rows`` (optional token indices) restricts the computation to those
    tokens and returns only their rows, in that order.  Each output row
    depends on its own token and the three before it, so sampled rows of a
    large input are exact.
    """
    T, H_qk, d = tuple(q_raw.shape)
    H_v = v_raw.shape[1]
    w = _as_np(conv_w).astype(np.float64).reshape((2 * H_qk + H_v) * d, 4)

    def rows_of(idx):  # raw rows [len(idx), C] in fp64, the q, k, v channels side by side
        return np.concatenate([_widen(q_raw[idx]).reshape(len(idx), -1),
                               _widen(k_raw[idx]).reshape(len(idx), -1),
                               _widen(v_raw[idx]).reshape(len(idx), -1)], axis=1)

    if cu_seqlens is None:
        cu = np.array([0, T])
    elif isinstance(cu_seqlens, (list, tuple)):
        cu = np.asarray(cu_seqlens, dtype=np.int64)
    else:
        cu = _as_np(cu_seqlens).astype(np.int64)
    if rows is None:
        sel = np.arange(T)
        y = causal_conv(rows_of(sel), w, cu)
    else:
        # only the sampled rows and the three before each are widened
        sel = np.asarray(rows, dtype=np.int64)
        y = np.zeros((len(sel), w.shape[0]))
        starts = cu[np.searchsorted(cu, sel, side="right") - 1]
        for r, (t, t0) in enumerate(zip(sel, starts)):
            taps = [t - 3 + i for i in range(4) if t - 3 + i >= t0]
            xs = rows_of(np.array(taps, dtype=np.int64))
            for j, tt in enumerate(taps):
                y[r] = y[r] + w[:, tt - t + 3] * xs[j]
    R = len(sel)
    y = _act(y, act)
    nq = H_qk * d
    q = _l2norm(y[:, :nq].reshape(R, H_qk, d), eps)
    k = _l2norm(y[:, nq:2 * nq].reshape(R, H_qk, d), eps)
    v = y[:, 2 * nq:].reshape(R, H_v, d)
    ad = _as_np(a).astype(np.float64)[sel]
    bd = _as_np(b).astype(np.float64)[sel]
    return q, k, v, -softplus(ad), sigmoid(bd)


def frontend_decode_step(q_raw, k_raw, v_raw, conv_w, a, b, conv_state, act="none", eps=1e-6):
    """One decode step of the front end for B sequences.

    ``conv_state [B, 3, C]`` holds each sequence's last three raw input rows
    (oldest first).  Returns ``(q, k, v, log_alpha, beta, new_state)``.
    """
    qr, kr, vr = _widen(q_raw), _widen(k_raw), _widen(v_raw)
    B, H_qk, d = qr.shape
    H_v = vr.shape[1]
    w = _as_np(conv_w).astype(np.float64).reshape((2 * H_qk + H_v) * d, 4)
    x = np.concatenate([qr.reshape(B, -1), kr.reshape(B, -1), vr.reshape(B, -1)], axis=1)
    st = _widen(conv_state)
    y = w[:, 0] * st[:, 0] + w[:, 1] * st[:, 1] + w[:, 2] * st[:, 2] + w[:, 3] * x
    y = _act(y, act)
    nq = H_qk * d
    q = _l2norm(y[:, :nq].reshape(B, H_qk, d), eps)
    k = _l2norm(y[:, nq:2 * nq].reshape(B, H_qk, d), eps)
    v = y[:, 2 * nq:].reshape(B, H_v, d)
    new_state = np.stack([st[:, 1], st[:, 2], x], axis=1)
    return (q, k, v, -softplus(_as_np(a).astype(np.float64)),
            sigmoid(_as_np(b).astype(np.float64)), new_state)
