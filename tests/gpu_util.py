"""Helpers shared by the GPU tests: error metrics of the acceptance bar.

The bar (bf16 q/k/v, fp32 gates and state) is
    max|o_gpu - o_ref| / max|o_ref|                <= 1e-2
    ||S_gpu - S_ref||_F / ||S_ref||_F               <= 1e-2
"""
import json
import os

import numpy as np
import torch

O_TOL = 1e-2
S_TOL = 1e-2


def o_err(o_gpu, o_ref, mask=None):
    a = o_gpu.float().cpu().double().numpy() if isinstance(o_gpu, torch.Tensor) else o_gpu
    b = np.asarray(o_ref, dtype=np.float64)
    if mask is not None:
        a, b = a[mask], b[mask]
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def s_err(S_gpu, S_ref, mask=None):
    a = S_gpu.cpu().double().numpy() if isinstance(S_gpu, torch.Tensor) else S_gpu
    b = np.asarray(S_ref, dtype=np.float64)
    if mask is not None:
        a, b = a[mask], b[mask]
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to_cuda(case):
    """Move a PrefillCase's tensors to the current CUDA device."""
    d = "cuda"
    return dict(q=case.q.to(d), k=case.k.to(d), v=case.v.to(d), log_alpha=case.log_alpha.to(d),
                beta=case.beta.to(d), S0=None if case.S0 is None else case.S0.to(d),
                cu_seqlens=case.cu_seqlens.to(d))


def record(test, workload, **errors):
    """Append one line of measured errors to the file named by GDN_PARITY_LOG
    (if set), so that a GPU run leaves a table of its parity margins."""
    path = os.environ.get("GDN_PARITY_LOG")
    if not path:
        return
    with open(path, "a") as f:
        f.write(json.dumps({"test": test, "workload": workload, **errors}) + "\n")


def per_head_o(o_gpu, o_ref, heads):
    """Worst o error of each listed value head (o is [T, H_v, d])."""
    a = o_gpu.float().cpu().double().numpy() if isinstance(o_gpu, torch.Tensor) else o_gpu
    return {int(h): o_err(a[:, h], np.asarray(o_ref)[:, h]) for h in heads}


def per_head_s(S_gpu, S_ref, heads):
    """Relative Frobenius S error of each listed value head (S is [N, H_v, d, d])."""
    a = S_gpu.cpu().double().numpy() if isinstance(S_gpu, torch.Tensor) else S_gpu
    return {int(h): s_err(a[:, h], np.asarray(S_ref)[:, h]) for h in heads}
