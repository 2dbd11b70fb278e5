"""fp64 CPU oracle for the Gated DeltaNet recurrence -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  It shares no code with the CUDA
library (``linear_attention_12_b200``) and never imports it.

Two independent formulations live here:

* :func:`prefill` / :func:`decode_step` / :func:`decode_multi` -- the sequential recurrence of the
  bjdmk.com.cn article "为什么 Qwen3.8-Flash-Next 值得单独跑一遍", section 2.1
  "Gated DeltaNet 负责廉价压缩历史" (state-update formula), evaluated token by
  token in plain C (``gdn_oracle.c``) in fp64, in its expanded "new value
  minus what the memory predicts" form, with readout ``o_t = S_t^T q_t``
  (post-update state, no scale; the pages give no readout, this is the plain
  reading).
* :func:`literal_prefill` -- the same formula taken literally: it builds the
  d_k x d_k matrix ``alpha_t (I - beta_t k_t k_t^T)`` and multiplies it into S
  with numpy.  Slow (O(d^3) per token); for tiny cases only.  It exists to pin
  the C oracle against a differently-written evaluation of the page's formula.

``oracle.backward`` holds the prefill's gradients (reverse mode of the same
recurrence, fp64 numpy); see its header.

``oracle.frontend`` holds the front end (short causal convolution, L2
normalisation of q and k, gate activations) in fp64 numpy; see its header.

Inputs are numpy arrays (or CPU torch tensors) in the library's layouts:
q, k ``[T, H_qk, dk]``; v ``[T, H_v, dv]`` (bf16 as uint16 bits, or float32);
log_alpha, beta ``[T, H_v]`` float32; S0 ``[N, H_v, dk, dv]`` float32 or None;
cu_seqlens ``[N+1]`` int32.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libgdn_oracle.so")

ORACLE_BF16 = 1
ORACLE_F32 = 2

_lock = threading.Lock()
_libs = {}


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the C oracle with gcc (default: ``oracle/_build``); return the path."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11", "-shared",
             "-fPIC", "-pthread", src, "-o", tmp, "-lm"])
        os.replace(tmp, out)
    return out


def _load(path=None):
    path = path or build()
    with _lock:
        lib = _libs.get(path)
        if lib is None:
            lib = ctypes.CDLL(path)
            lib.gdn_oracle_run.restype = ctypes.c_int
            lib.gdn_oracle_run.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_void_p, ctypes.c_int,
                ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
            _libs[path] = lib
    return lib


def _as_np(x):
    """CPU torch tensor or numpy array -> contiguous numpy array (bf16 -> uint16 bits)."""
    if x is None:
        return None
    if not isinstance(x, np.ndarray):  # torch tensor
        import torch
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            x = x.view(torch.int16).numpy().view(np.uint16)
        else:
            x = x.numpy()
    return np.ascontiguousarray(x)


def _io_dtype(arr: np.ndarray) -> int:
    if arr.dtype == np.uint16:
        return ORACLE_BF16
    if arr.dtype == np.float32:
        return ORACLE_F32
    raise TypeError(f"oracle inputs must be bf16 bits (uint16) or float32, got {arr.dtype}")


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def run_units(q, k, v, log_alpha, beta, units, S_init=None, want_o=True, n_threads=None,
              lib=None):
    """Run the recurrence on explicit units.

    ``units`` is an int array ``[n, 3]`` of (t0, t1, h).  Returns
    ``(S_out [n, dk, dv] fp64, o list of [t1-t0, dv] fp64 arrays or None)``.
    ``lib`` selects another build of the C oracle (used by the tests that plant
    mistakes in a copy of it).
    """
    q, k, v = _as_np(q), _as_np(k), _as_np(v)
    la = np.ascontiguousarray(_as_np(log_alpha), dtype=np.float32)
    be = np.ascontiguousarray(_as_np(beta), dtype=np.float32)
    dt = _io_dtype(q)
    assert _io_dtype(k) == dt and _io_dtype(v) == dt, "q, k, v must share one dtype"
    T, H_qk, dk = q.shape
    Tv, H_v, dv = v.shape
    assert k.shape == q.shape and Tv == T and la.shape == (T, H_v) and be.shape == (T, H_v)
    units = np.ascontiguousarray(np.asarray(units, dtype=np.int32).reshape(-1, 3))
    n = units.shape[0]
    S_out = np.empty((n, dk, dv), dtype=np.float64)
    S_in = None
    if S_init is not None:
        S_in = np.ascontiguousarray(np.asarray(S_init, dtype=np.float64).reshape(n, dk, dv))
    o_out = offs = None
    if want_o:
        lens = (units[:, 1] - units[:, 0]).astype(np.int64)
        offs = np.zeros(n, dtype=np.int64)
        if n > 1:
            offs[1:] = np.cumsum(lens)[:-1]
        o_out = np.empty((int(lens.sum()), dv), dtype=np.float64)
    ptr = lambda a: None if a is None else a.ctypes.data
    rc = _load(lib).gdn_oracle_run(
        ptr(q), ptr(k), ptr(v), dt, ptr(la), ptr(be), T, H_qk, H_v, dk, dv,
        ptr(units), n, ptr(S_in), ptr(S_out), ptr(o_out), ptr(offs),
        int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError("gdn_oracle_run rejected its arguments")
    o_list = None
    if want_o:
        o_list = [o_out[offs[i]: offs[i] + (units[i, 1] - units[i, 0])] for i in range(n)]
    return S_out, o_list


def prefill(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, heads=None,
            want_o=True, n_threads=None, lib=None):
    """Sequential fp64 prefill over packed sequences.

    Returns ``(o, S_final)``: ``o`` is ``[T, H_v, dv]`` fp64 (NaN for heads not
    requested; None when ``want_o`` is False) and ``S_final`` is
    ``[N, H_v, dk, dv]`` fp64 (NaN for heads not requested).  ``heads`` limits
    the work to a subset of value heads (for sampled checks of large cases).
    """
    qn = _as_np(q)
    T, H_qk, dk = qn.shape
    vn = _as_np(v)
    H_v, dv = vn.shape[1], vn.shape[2]
    cu = np.array([0, T], dtype=np.int64) if cu_seqlens is None else _as_np(cu_seqlens).astype(np.int64)
    N = len(cu) - 1
    heads = list(range(H_v)) if heads is None else [int(h) for h in heads]
    units = [(int(cu[n]), int(cu[n + 1]), h) for n in range(N) for h in heads]
    S_init = None
    if S0 is not None:
        S0n = _as_np(S0)
        S_init = np.stack([S0n[n, h] for n in range(N) for h in heads]).astype(np.float64)
    S_out, o_list = run_units(qn, _as_np(k), vn, log_alpha, beta, units, S_init, want_o,
                              n_threads, lib)
    S_final = np.full((N, H_v, dk, dv), np.nan)
    o = np.full((T, H_v, dv), np.nan) if want_o else None
    i = 0
    for n in range(N):
        for h in heads:
            S_final[n, h] = S_out[i]
            if want_o:
                o[cu[n]:cu[n + 1], h] = o_list[i]
            i += 1
    return o, S_final


def decode_step(q, k, v, log_alpha, beta, S, units_bh=None, n_threads=None):
    """One decode step for a batch: q, k ``[B, H_qk, dk]``, v ``[B, H_v, dv]``,
    gates ``[B, H_v]``, S ``[B, H_v, dk, dv]``.  Returns ``(o [B,H_v,dv], S_new)``
    in fp64.  With ``units_bh`` (a list of (b, h) pairs) only those units are
    advanced: S is then ``[len(units_bh), dk, dv]`` (one state per pair) and the
    returned arrays hold one row per pair, in that order.
    """
    qn = _as_np(q)
    B = qn.shape[0]
    vn = _as_np(v)
    H_v, dv = vn.shape[1], vn.shape[2]
    Sn = np.asarray(_as_np(S), dtype=np.float64)
    if units_bh is None:
        pairs = [(b, h) for b in range(B) for h in range(H_v)]
        S_init = Sn.reshape(B * H_v, *Sn.shape[2:])
    else:
        pairs = [(int(b), int(h)) for (b, h) in units_bh]
        S_init = Sn
    units = [(b, b + 1, h) for (b, h) in pairs]
    S_out, o_list = run_units(qn, _as_np(k), vn, log_alpha, beta, units, S_init, True, n_threads)
    o = np.stack([x[0] for x in o_list])
    if units_bh is None:
        return o.reshape(B, H_v, dv), S_out.reshape(B, H_v, *S_out.shape[1:])
    return o, S_out


def decode_multi(q, k, v, log_alpha, beta, S, n_threads=None):
    """M decode steps per sequence, taken in order (speculative verification of
    1 + k drafted tokens): q, k ``[B, M, H_qk, dk]``, v ``[B, M, H_v, dv]``,
    gates ``[B, M, H_v]``, S ``[B, H_v, dk, dv]``.

    Token j of every sequence is one application of the state-update formula
    to the state left by token j - 1, i.e. :func:`decode_step` called M times.
    Returns ``(o [B, M, H_v, dv], S_steps [B, M, H_v, dk, dv])`` in fp64, where
    ``S_steps[:, j]`` is the state after token j (the state to keep when the
    first j + 1 tokens are accepted).
    """
    qn, kn, vn = _as_np(q), _as_np(k), _as_np(v)
    la, be = _as_np(log_alpha), _as_np(beta)
    M = qn.shape[1]
    state = S
    outs, states = [], []
    for j in range(M):
        o_j, state = decode_step(qn[:, j], kn[:, j], vn[:, j], la[:, j], be[:, j], state,
                                 n_threads=n_threads)
        outs.append(o_j)
        states.append(state)
    return np.stack(outs, axis=1), np.stack(states, axis=1)


def _widen(x) -> np.ndarray:
    a = _as_np(x)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def literal_prefill(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None):
    """The state-update formula taken literally, for tiny sizes only.

    For each token it forms the d_k x d_k matrix ``alpha (I - beta k k^T)``
    explicitly and computes ``S <- M @ S + beta * outer(k, v)``, then
    ``o = S^T q``.  Written independently of ``gdn_oracle.c``.
    """
    qd, kd, vd = _widen(q), _widen(k), _widen(v)
    la = _as_np(log_alpha).astype(np.float64)
    be = _as_np(beta).astype(np.float64)
    T, H_qk, dk = qd.shape
    H_v, dv = vd.shape[1], vd.shape[2]
    group = H_v // H_qk
    cu = np.array([0, T]) if cu_seqlens is None else _as_np(cu_seqlens).astype(np.int64)
    N = len(cu) - 1
    o = np.zeros((T, H_v, dv))
    S_final = np.zeros((N, H_v, dk, dv))
    eye = np.eye(dk)
    for n in range(N):
        for h in range(H_v):
            S = np.zeros((dk, dv)) if S0 is None else _as_np(S0)[n, h].astype(np.float64)
            for t in range(cu[n], cu[n + 1]):
                kt = kd[t, h // group]
                a, b = np.exp(la[t, h]), be[t, h]
                M = a * (eye - b * np.outer(kt, kt))
                S = M @ S + b * np.outer(kt, vd[t, h])
                o[t, h] = S.T @ qd[t, h // group]
            S_final[n, h] = S
    return o, S_final
