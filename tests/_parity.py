"""Helpers shared by the GPU parity tests: error metrics and unit slicing.

Tolerances (stated for the method: the gated delta rule on one B200):
  fp32 inputs:  per tensor  max|x - ref| / max|ref|  <= 1e-4
  bf16 inputs with fp32 state:  per tensor  max|x - ref| / rms(ref)  <= 2e-2
"""
from __future__ import annotations

import numpy as np
import torch

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def to64(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def rel_max(x, ref):
    x, ref = to64(x), to64(ref)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-30))


def rel_rms(x, ref):
    x, ref = to64(x), to64(ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.max(np.abs(x - ref)) / max(rms, 1e-30))


def metric_for(dtype):
    return (rel_max, TOL_F32) if dtype == torch.float32 else (rel_rms, TOL_BF16)


def unit_slice(p, n, h):
    """Inputs of one (sequence n, v-head h) unit as a single-head problem (CPU tensors)."""
    Hqk, Hv = p.q.shape[2], p.v.shape[2]
    hq = h // (Hv // Hqk)
    if p.cu_seqlens is not None:
        cu = p.cu_seqlens.tolist()
        b, t0, t1 = 0, cu[n], cu[n + 1]
    else:
        b, t0, t1 = n, 0, p.q.shape[1]
    sl = lambda x, hh: None if x is None else x[b:b + 1, t0:t1, hh:hh + 1]
    st = None if p.state_in is None else p.state_in[n:n + 1, h:h + 1]
    g = None if p.g is None else p.g[b:b + 1, t0:t1, h:h + 1]
    return (sl(p.q, hq), sl(p.k, hq), sl(p.v, h), g, p.beta[b:b + 1, t0:t1, h:h + 1], st), (b, t0, t1)
