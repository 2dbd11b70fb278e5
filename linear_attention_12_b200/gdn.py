"""ctypes binding of ``libgdn.so`` (C ABI in ``include/gdn.h``).

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch provides device memory and the current stream.  There is no
fallback: if the library is missing, or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_OK = 0
GDN_ERR_INVALID_ARG = 1
GDN_ERR_UNSUPPORTED = 2
GDN_ERR_CUDA = 3
GDN_ERR_TIMEOUT = 4
GDN_ERR_WORKSPACE = 5
GDN_BF16 = 1
GDN_F32 = 2
GDN_ACT_NONE = 0
GDN_ACT_SILU = 1
_ACTS = {"none": GDN_ACT_NONE, "silu": GDN_ACT_SILU}

# Every exported symbol of include/gdn.h with its ctypes signature.
_c = ctypes
SIGNATURES = {
    "gdn_prefill": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                               _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_int32, _c.c_int32,
                               _c.c_int32, _c.c_int32, _c.c_int32, _c.c_int, _c.c_void_p,
                               _c.c_void_p, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "gdn_prefill_workspace_size": (_c.c_size_t, [_c.c_int32] * 6 + [_c.c_int]),
    "gdn_prefill_mma": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                   _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_int32, _c.c_int32,
                                   _c.c_int32, _c.c_int32, _c.c_int32, _c.c_int, _c.c_void_p,
                                   _c.c_void_p, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "gdn_prefill_tc": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                  _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_int32, _c.c_int32,
                                  _c.c_int32, _c.c_int32, _c.c_int32, _c.c_int, _c.c_void_p,
                                  _c.c_void_p, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "gdn_prefill_segmented": (_c.c_int, [_c.c_void_p] * 7 + [_c.c_int32] * 6 +
                              [_c.c_int, _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_void_p,
                               _c.c_size_t, _c.c_void_p]),
    "gdn_prefill_segmented_workspace_size": (_c.c_size_t,
                                             [_c.c_int32] * 6 + [_c.c_int, _c.c_int32]),
    "gdn_prefill_auto_segments": (_c.c_int32, [_c.c_int32] * 4),
    "gdn_prefill_backward": (_c.c_int, [_c.c_void_p] * 9 + [_c.c_int32] * 6 +
                             [_c.c_int] + [_c.c_void_p] * 7 + [_c.c_size_t, _c.c_void_p]),
    "gdn_prefill_backward_saved": (_c.c_int, [_c.c_void_p] * 9 + [_c.c_int32] * 6 +
                                   [_c.c_int] + [_c.c_void_p] * 7 + [_c.c_size_t, _c.c_void_p]),
    "gdn_prefill_train": (_c.c_int, [_c.c_void_p] * 7 + [_c.c_int32] * 6 +
                          [_c.c_int, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                           _c.c_void_p]),
    "gdn_prefill_backward_workspace_size": (_c.c_size_t, [_c.c_int32] * 6 + [_c.c_int]),
    "gdn_prefill_noalloc": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                       _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int32,
                                       _c.c_int32, _c.c_int32, _c.c_int32, _c.c_int32,
                                       _c.c_int32, _c.c_int, _c.c_void_p, _c.c_void_p,
                                       _c.c_void_p]),
    "gdn_prefill_noalloc_max_scratch_bytes": (_c.c_size_t, []),
    "gdn_decode_step": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                   _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_int32, _c.c_int32,
                                   _c.c_int32, _c.c_int32, _c.c_int, _c.c_void_p, _c.c_void_p]),
    "gdn_decode_multi": (_c.c_int, [_c.c_void_p] * 6 + [_c.c_int32] * 6 + [_c.c_int, _c.c_void_p,
                                                                          _c.c_void_p, _c.c_void_p]),
    "gdn_frontend": (_c.c_int, [_c.c_void_p] * 7 + [_c.c_int32] * 6 + [_c.c_int, _c.c_int,
                                                                         _c.c_float] +
                     [_c.c_void_p] * 6),
    "gdn_frontend_decode_step": (_c.c_int, [_c.c_void_p] * 7 + [_c.c_int32] * 5 +
                                 [_c.c_int, _c.c_int, _c.c_float] + [_c.c_void_p] * 6),
    "gdn_get_last_device_error": (_c.c_int, [_c.c_void_p]),
    "gdn_selftest_bounded_wait": (_c.c_int, [_c.c_void_p]),
    "gdn_status_string": (_c.c_char_p, [_c.c_int]),
    "gdn_version": (_c.c_int32, []),
}

_lock = threading.Lock()
_lib = None


class GDNError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """Load ``libgdn.so`` (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m linear_attention_12_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdn_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _io_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _check(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def workspace_size(N, T, H_qk, H_v, d=128, io_dtype=GDN_BF16, segments=0) -> int:
    return int(lib().gdn_prefill_segmented_workspace_size(N, T, H_qk, H_v, d, d, io_dtype,
                                                          segments))


MAX_PREFILL_SEGMENTS = 64  # GDN_MAX_PREFILL_SEGMENTS


def auto_segments(N, T, H_qk, H_v) -> int:
    """Segments per sequence ``prefill`` uses for these sizes on the current device."""
    return int(lib().gdn_prefill_auto_segments(N, T, H_qk, H_v))


def prefill(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, o=None, S_final=None,
            want_state=True, workspace=None, segments=None, state_pass="auto", stream=None):
    """Chunked prefill.  Returns ``(o, S_final)`` (``S_final`` None if not wanted).

    ``segments``: None or 0 lets the library split long sequences when that
    fills more SMs; 1 disables the split; 2 .. 64 forces that many pieces per
    sequence (gdn_prefill_segmented).  ``state_pass``: "auto" (the library's
    choice per slice width), "tcgen05" (gdn_prefill_tc) or "mma_sync"
    (gdn_prefill_mma); the last two take the automatic segment choice only."""
    T, H_qk, dk = q.shape
    H_v, dv = v.shape[1], v.shape[2]
    dt = q.dtype
    _check(q, "q", dt)
    _check(k, "k", dt, q.shape)
    _check(v, "v", dt, (T, H_v, dv))
    _check(log_alpha, "log_alpha", torch.float32, (T, H_v))
    _check(beta, "beta", torch.float32, (T, H_v))
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32, device=q.device)
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    N = cu_seqlens.numel() - 1
    if S0 is not None:
        _check(S0, "S0", torch.float32, (N, H_v, dk, dv))
    if o is None:
        o = torch.empty((T, H_v, dv), dtype=dt, device=q.device)
    _check(o, "o", dt, (T, H_v, dv))
    if S_final is None and want_state:
        S_final = torch.empty((N, H_v, dk, dv), dtype=torch.float32, device=q.device)
    if S_final is not None:
        _check(S_final, "S_final", torch.float32, (N, H_v, dk, dv))
    io = _io_dtype(q)
    seg = 0 if segments is None else int(segments)
    need = workspace_size(N, T, H_qk, H_v, dk, io, segments=seg)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if state_pass not in ("auto", "tcgen05", "mma_sync"):
        raise ValueError(f"state_pass: 'auto', 'tcgen05' or 'mma_sync', not {state_pass!r}")
    if state_pass != "auto":
        if seg != 0:
            raise ValueError("a fixed state_pass takes the automatic segment choice only")
        fn = lib().gdn_prefill_tc if state_pass == "tcgen05" else lib().gdn_prefill_mma
        st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                _ptr(cu_seqlens), N, T, H_qk, H_v, dk, dv, io, _ptr(o), _ptr(S_final),
                _ptr(workspace), wbytes, _stream_handle(stream))
    else:
        st = lib().gdn_prefill_segmented(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                         _ptr(S0), _ptr(cu_seqlens), N, T, H_qk, H_v, dk, dv, io,
                                         _ptr(o), _ptr(S_final), seg, _ptr(workspace), wbytes,
                                         _stream_handle(stream))
    if st != GDN_OK:
        raise GDNError(st, {"auto": "gdn_prefill_segmented", "tcgen05": "gdn_prefill_tc",
                            "mma_sync": "gdn_prefill_mma"}[state_pass])
    return o, S_final


def decode_step(q, k, v, log_alpha, beta, S, *, o=None, stream=None):
    """One decode step; ``S`` [B, H_v, dk, dv] fp32 is updated in place.  Returns ``o``."""
    B, H_qk, dk = q.shape
    H_v, dv = v.shape[1], v.shape[2]
    dt = q.dtype
    _check(q, "q", dt)
    _check(k, "k", dt, q.shape)
    _check(v, "v", dt, (B, H_v, dv))
    _check(log_alpha, "log_alpha", torch.float32, (B, H_v))
    _check(beta, "beta", torch.float32, (B, H_v))
    _check(S, "S", torch.float32, (B, H_v, dk, dv))
    if o is None:
        o = torch.empty((B, H_v, dv), dtype=dt, device=q.device)
    _check(o, "o", dt, (B, H_v, dv))
    st = lib().gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S),
                               B, H_qk, H_v, dk, dv, _io_dtype(q), _ptr(o),
                               _stream_handle(stream))
    if st != GDN_OK:
        raise GDNError(st, "gdn_decode_step")
    return o


def backward_workspace(q, v, cu_seqlens=None):
    """A workspace tensor of gdn_prefill_backward_workspace_size bytes for these inputs
    (also what ``prefill_train`` fills)."""
    T, H_qk, dk_ = q.shape
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    need = int(lib().gdn_prefill_backward_workspace_size(N, T, H_qk, v.shape[1], dk_,
                                                         v.shape[2], _io_dtype(q)))
    return torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)


def prefill_train(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, o=None, S_final=None,
                  workspace=None, stream=None):
    """The prefill of a training step (gdn_prefill_train): returns ``(o, S_final,
    workspace)``, the workspace holding what ``prefill_backward(..., saved=True)``
    reads for the same inputs."""
    T, H_qk, dk_ = q.shape
    H_v, dv_ = v.shape[1], v.shape[2]
    dt = q.dtype
    _check(q, "q", dt)
    _check(k, "k", dt, q.shape)
    _check(v, "v", dt, (T, H_v, dv_))
    _check(log_alpha, "log_alpha", torch.float32, (T, H_v))
    _check(beta, "beta", torch.float32, (T, H_v))
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32, device=q.device)
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    N = cu_seqlens.numel() - 1
    if S0 is not None:
        _check(S0, "S0", torch.float32, (N, H_v, dk_, dv_))
    if o is None:
        o = torch.empty((T, H_v, dv_), dtype=dt, device=q.device)
    _check(o, "o", dt, (T, H_v, dv_))
    if S_final is None:
        S_final = torch.empty((N, H_v, dk_, dv_), dtype=torch.float32, device=q.device)
    _check(S_final, "S_final", torch.float32, (N, H_v, dk_, dv_))
    if workspace is None:
        workspace = backward_workspace(q, v, cu_seqlens)
    wbytes = workspace.numel() * workspace.element_size()
    st = lib().gdn_prefill_train(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                 _ptr(S0), _ptr(cu_seqlens), N, T, H_qk, H_v, dk_, dv_,
                                 _io_dtype(q), _ptr(o), _ptr(S_final), _ptr(workspace), wbytes,
                                 _stream_handle(stream))
    if st != GDN_OK:
        raise GDNError(st, "gdn_prefill_train")
    return o, S_final, workspace


def prefill_backward(q, k, v, log_alpha, beta, dO, S0=None, dS_final=None, cu_seqlens=None, *,
                     want_dS0=True, workspace=None, saved=False, stream=None):
    """Gradients of ``L = <dO, o> + <dS_final, S_final>`` for gdn_prefill (bf16 or
    fp32 q, k, v, dO; the gradients of q, k, v in the same type).  ``saved=True``:
    ``workspace`` is the one ``prefill_train`` filled for the same inputs, and the
    forward pass is not re-run (gdn_prefill_backward_saved).

    Returns ``(dq, dk, dv, dlog_alpha, dbeta, dS0)`` (``dS0`` None if not wanted)."""
    if saved and workspace is None:
        raise ValueError("saved=True needs the workspace prefill_train filled")
    T, H_qk, dk_ = q.shape
    H_v, dv_ = v.shape[1], v.shape[2]
    dt = q.dtype
    _check(q, "q", dt)
    _check(k, "k", dt, q.shape)
    _check(v, "v", dt, (T, H_v, dv_))
    _check(dO, "dO", dt, (T, H_v, dv_))
    _check(log_alpha, "log_alpha", torch.float32, (T, H_v))
    _check(beta, "beta", torch.float32, (T, H_v))
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32, device=q.device)
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    N = cu_seqlens.numel() - 1
    if S0 is not None:
        _check(S0, "S0", torch.float32, (N, H_v, dk_, dv_))
    if dS_final is not None:
        _check(dS_final, "dS_final", torch.float32, (N, H_v, dk_, dv_))
    dq, dk = torch.empty_like(q), torch.empty_like(k)
    dv = torch.empty_like(v)
    dla, dbe = torch.empty_like(log_alpha), torch.empty_like(beta)
    dS0 = (torch.empty((N, H_v, dk_, dv_), dtype=torch.float32, device=q.device)
           if want_dS0 else None)
    io = _io_dtype(q)
    need = int(lib().gdn_prefill_backward_workspace_size(N, T, H_qk, H_v, dk_, dv_, io))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fn = lib().gdn_prefill_backward_saved if saved else lib().gdn_prefill_backward
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
            _ptr(cu_seqlens), _ptr(dO), _ptr(dS_final), N, T, H_qk, H_v, dk_, dv_, io, _ptr(dq),
            _ptr(dk), _ptr(dv), _ptr(dla), _ptr(dbe), _ptr(dS0), _ptr(workspace), wbytes,
            _stream_handle(stream))
    if st != GDN_OK:
        raise GDNError(st, "gdn_prefill_backward_saved" if saved else "gdn_prefill_backward")
    return dq, dk, dv, dla, dbe, dS0


MAX_DECODE_TOKENS = 8  # GDN_MAX_DECODE_TOKENS


def decode_multi(q, k, v, log_alpha, beta, S_in, *, o=None, S_steps=None, stream=None):
    """M tokens per sequence in one pass over the state (speculative verification).

    q, k [B, M, H_qk, dk], v [B, M, H_v, dv], gates [B, M, H_v], S_in
    [B, H_v, dk, dv] fp32 (read only).  Returns ``(o [B, M, H_v, dv],
    S_steps [B, M, H_v, dk, dv])`` where ``S_steps[:, j]`` is the state after
    token j."""
    B, M, H_qk, dk = q.shape
    H_v, dv = v.shape[2], v.shape[3]
    dt = q.dtype
    _check(q, "q", dt)
    _check(k, "k", dt, q.shape)
    _check(v, "v", dt, (B, M, H_v, dv))
    _check(log_alpha, "log_alpha", torch.float32, (B, M, H_v))
    _check(beta, "beta", torch.float32, (B, M, H_v))
    _check(S_in, "S_in", torch.float32, (B, H_v, dk, dv))
    if o is None:
        o = torch.empty((B, M, H_v, dv), dtype=dt, device=q.device)
    if S_steps is None:
        S_steps = torch.empty((B, M, H_v, dk, dv), dtype=torch.float32, device=q.device)
    _check(o, "o", dt, (B, M, H_v, dv))
    _check(S_steps, "S_steps", torch.float32, (B, M, H_v, dk, dv))
    st = lib().gdn_decode_multi(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                _ptr(S_in), B, M, H_qk, H_v, dk, dv, _io_dtype(q), _ptr(o),
                                _ptr(S_steps), _stream_handle(stream))
    if st != GDN_OK:
        raise GDNError(st, "gdn_decode_multi")
    return o, S_steps


def frontend(q_raw, k_raw, v_raw, conv_w, a, b, cu_seqlens=None, *, act="none", eps=1e-6,
             out=None, stream=None):
    """Short causal convolution, q/k L2 normalisation and gate activations.

    Returns ``(q, k, v, log_alpha, beta)`` -- gdn_prefill's inputs.  ``out``
    may supply those five tensors."""
    T, H_qk, dk = q_raw.shape
    H_v, dv = v_raw.shape[1], v_raw.shape[2]
    dt = q_raw.dtype
    _check(q_raw, "q_raw", dt)
    _check(k_raw, "k_raw", dt, q_raw.shape)
    _check(v_raw, "v_raw", dt, (T, H_v, dv))
    _check(conv_w, "conv_w", torch.float32, ((2 * H_qk + H_v) * dk, 4))
    _check(a, "a", torch.float32, (T, H_v))
    _check(b, "b", torch.float32, (T, H_v))
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32, device=q_raw.device)
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    N = cu_seqlens.numel() - 1
    if out is None:
        out = (torch.empty_like(q_raw), torch.empty_like(k_raw), torch.empty_like(v_raw),
               torch.empty_like(a), torch.empty_like(b))
    q, k, v, la, be = out
    for t, ref, name in ((q, q_raw, "q"), (k, k_raw, "k"), (v, v_raw, "v")):
        _check(t, name, dt, ref.shape)
    _check(la, "log_alpha", torch.float32, (T, H_v))
    _check(be, "beta", torch.float32, (T, H_v))
    st = lib().gdn_frontend(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_w), _ptr(a), _ptr(b),
                            _ptr(cu_seqlens), N, T, H_qk, H_v, dk, dv, _io_dtype(q_raw),
                            _ACTS[act], float(eps), _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be),
                            _stream_handle(stream))
    if st != GDN_OK:
        raise GDNError(st, "gdn_frontend")
    return q, k, v, la, be


def frontend_decode_step(q_raw, k_raw, v_raw, conv_w, a, b, conv_state, *, act="none", eps=1e-6,
                         stream=None):
    """One decode step of the front end; ``conv_state`` [B, 3, C] is shifted in
    place.  Returns ``(q, k, v, log_alpha, beta)``."""
    B, H_qk, dk = q_raw.shape
    H_v, dv = v_raw.shape[1], v_raw.shape[2]
    dt = q_raw.dtype
    _check(q_raw, "q_raw", dt)
    _check(k_raw, "k_raw", dt, q_raw.shape)
    _check(v_raw, "v_raw", dt, (B, H_v, dv))
    _check(conv_w, "conv_w", torch.float32, ((2 * H_qk + H_v) * dk, 4))
    _check(a, "a", torch.float32, (B, H_v))
    _check(b, "b", torch.float32, (B, H_v))
    _check(conv_state, "conv_state", dt, (B, 3, (2 * H_qk + H_v) * dk))
    q, k, v = torch.empty_like(q_raw), torch.empty_like(k_raw), torch.empty_like(v_raw)
    la, be = torch.empty_like(a), torch.empty_like(b)
    st = lib().gdn_frontend_decode_step(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_w),
                                        _ptr(a), _ptr(b), _ptr(conv_state), B, H_qk, H_v, dk, dv,
                                        _io_dtype(q_raw), _ACTS[act], float(eps), _ptr(q),
                                        _ptr(k), _ptr(v), _ptr(la), _ptr(be),
                                        _stream_handle(stream))
    if st != GDN_OK:
        raise GDNError(st, "gdn_frontend_decode_step")
    return q, k, v, la, be


def selftest_bounded_wait(stream=None) -> None:
    """Enqueue the library's bounded-wait self-test (a wait that runs out)."""
    st = lib().gdn_selftest_bounded_wait(_stream_handle(stream))
    if st != GDN_OK:
        raise GDNError(st, "gdn_selftest_bounded_wait")


def last_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status."""
    return int(lib().gdn_get_last_device_error(_stream_handle(stream)))
