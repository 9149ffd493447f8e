"""B200 gated delta rule: thin Python binding over the C ABI of ``libdr.so``.

This module only marshals arguments: it checks tensor placement, dtype and
contiguity, allocates outputs with PyTorch (device memory and streams are the
only things PyTorch does here) and passes raw device pointers plus the current
CUDA stream to the library's calls (``include/dr.h``).  Every step runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and a missing or
unloadable ``libdr.so`` raises.

    o, state_out = chunk_fwd(q, k, v, g, beta, state_in=None, cu_seqlens=None)
    o = recurrent_step(q, k, v, g, beta, state)      # state updated in place
    y, conv_state = short_conv_silu(x, w)            # the step before the rule
    out = norm_gate(o, weight, z=z)                  # the step after it
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

__all__ = ["chunk_fwd", "recurrent_step", "short_conv_silu", "norm_gate", "device_status",
           "prefill_kernel", "chunk_state_rows", "lib", "DrError", "LIB_PATH", "CHUNK"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdr.so")

DR_F32, DR_BF16 = 0, 1
_DTYPES = {torch.float32: DR_F32, torch.bfloat16: DR_BF16}
STATUS = {0: "DR_OK", 1: "DR_ERR_NULL", 2: "DR_ERR_SHAPE", 3: "DR_ERR_DTYPE", 4: "DR_ERR_ALIGN",
          5: "DR_ERR_UNSUPPORTED", 6: "DR_ERR_CUDA", 7: "DR_ERR_TIMEOUT"}

_lib = None


class DrError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({_status_string(code)})")


def lib() -> ctypes.CDLL:
    """Load ``libdr.so`` (built in-tree by ``gated_delta_rule_59_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m gated_delta_rule_59_b200.build` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        vp, fp, ip, i32 = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32
        L.dr_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, ip, i32, i32, i32, i32, i32, i32, i32,
                                   ctypes.c_int, ctypes.c_float, vp, ctypes.c_int, fp, fp,
                                   ctypes.c_uint32, vp]
        L.dr_chunk_fwd.restype = ctypes.c_int
        L.dr_short_conv_silu.argtypes = [vp, ctypes.c_int, fp, i32, fp, fp, ip, i32, i32, i32,
                                         i32, vp, ctypes.c_int, vp]
        L.dr_short_conv_silu.restype = ctypes.c_int
        L.dr_norm_gate.argtypes = [vp, ctypes.c_int, fp, fp, vp, ctypes.c_int, ctypes.c_int64,
                                   i32, i32, ctypes.c_float, vp, ctypes.c_int, vp]
        L.dr_norm_gate.restype = ctypes.c_int
        L.dr_recurrent_step.argtypes = [vp, vp, vp, fp, fp, fp, i32, i32, i32, i32, i32,
                                        ctypes.c_int, ctypes.c_float, vp, ctypes.c_int,
                                        ctypes.c_uint32, vp]
        L.dr_recurrent_step.restype = ctypes.c_int
        L.dr_status_string.argtypes = [ctypes.c_int]
        L.dr_status_string.restype = ctypes.c_char_p
        L.dr_get_device_status.argtypes = [vp]
        L.dr_get_device_status.restype = ctypes.c_int
        L.dr_version.restype = ctypes.c_int32
        L.dr_chunk_fwd_kernel.argtypes = [ctypes.c_int, ctypes.c_int32, ctypes.c_int32]
        L.dr_chunk_fwd_kernel.restype = ctypes.c_int
        _lib = L
    return _lib


def _status_string(code: int) -> str:
    try:
        return lib().dr_status_string(code).decode()
    except Exception:  # pragma: no cover - only while the library fails to load
        return "?"


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t: Optional[torch.Tensor], name: str, dtype=None, device=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


CHUNK = 64  # DR_CHUNK of include/dr.h: tokens between two returned chunk states


def chunk_state_rows(cu_seqlens, B: int, T: int) -> int:
    """Rows of the ``chunk_states`` output: ceil(max(len, 0) / CHUNK) per sequence.

    ``cu_seqlens`` (a tensor or sequence, or None for B sequences of T tokens) is read on
    the host; a device tensor is copied over (one synchronisation).
    """
    if cu_seqlens is None:
        return B * (-(-T // CHUNK))
    cu = cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else list(cu_seqlens)
    return sum(-(-max(int(b) - int(a), 0) // CHUNK) for a, b in zip(cu[:-1], cu[1:]))


def chunk_fwd(q, k, v, g, beta, state_in=None, cu_seqlens=None, scale: float = 1.0,
              output_final_state: bool = True, out_dtype=torch.float32, o=None, state_out=None,
              qk_l2norm: bool = False, output_chunk_states: bool = False, chunk_states=None):
    """Chunked prefill through ``dr_chunk_fwd``.

    q, k [B, T, Hqk, dk] and v [B, T, Hv, dv] in bf16 or fp32 (same dtype);
    g (or None), beta [B, T, Hv] fp32; state_in [N, Hv, dk, dv] fp32 or None;
    g may be [B, T, Hv, dk] instead: one log decay per key channel (``DR_GATE_PER_CHANNEL``,
    the "linear_attention" page's ChannelGates), run by the CUDA-core kernel.
    cu_seqlens int32 [N+1] (device) or None.  ``qk_l2norm``: the kernel divides every q and
    k row by its L2 norm first (``DR_QK_L2NORM``).  Returns (o [B, T, Hv, dv] in
    ``out_dtype``, state_out [N, Hv, dk, dv] fp32 or None).
    ``output_chunk_states`` (or a given ``chunk_states`` tensor): a third output holds the
    state after every ``CHUNK`` tokens of each sequence and after its last token,
    [chunk_state_rows(cu_seqlens, B, T), Hv, dk, dv] fp32, sequence after sequence.
    Allocating it with cu_seqlens reads cu_seqlens on the host.
    """
    if q.dtype not in _DTYPES or out_dtype not in _DTYPES:
        raise ValueError("q/k/v must be bf16 or fp32; out_dtype bf16 or fp32")
    dev = q.device
    _check(q, "q", q.dtype, dev)
    _check(k, "k", q.dtype, dev)
    _check(v, "v", q.dtype, dev)
    _check(g, "g", torch.float32, dev)
    _check(beta, "beta", torch.float32, dev)
    _check(state_in, "state_in", torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if k.shape != q.shape or v.shape[:2] != (B, T) or beta.shape != (B, T, Hv):
        raise ValueError("inconsistent shapes")
    channel_gates = g is not None and g.dim() == 4
    if g is not None and tuple(g.shape) not in ((B, T, Hv), (B, T, Hv, dk)):
        raise ValueError("g must be [B, T, Hv] or [B, T, Hv, dk]")
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if state_in is not None and tuple(state_in.shape) != (N, Hv, dk, dv):
        raise ValueError(f"state_in must be {(N, Hv, dk, dv)}")
    if o is None:
        o = torch.empty((B, T, Hv, dv), dtype=out_dtype, device=dev)
    _check(o, "o", out_dtype, dev)
    if output_final_state and state_out is None:
        state_out = torch.empty((N, Hv, dk, dv), dtype=torch.float32, device=dev)
    _check(state_out, "state_out", torch.float32, dev)
    want_cs = output_chunk_states or chunk_states is not None
    if want_cs:
        rows = chunk_state_rows(cu_seqlens, B, T)
        if chunk_states is None:
            chunk_states = torch.empty((rows, Hv, dk, dv), dtype=torch.float32, device=dev)
        elif tuple(chunk_states.shape) != (rows, Hv, dk, dv):
            raise ValueError(f"chunk_states must be {(rows, Hv, dk, dv)}")
        _check(chunk_states, "chunk_states", torch.float32, dev)
    rc = lib().dr_chunk_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in), _ptr(cu_seqlens), N,
        B, T, Hqk, Hv, dk, dv, _DTYPES[q.dtype], float(scale), _ptr(o), _DTYPES[out_dtype],
        _ptr(state_out), _ptr(chunk_states) if want_cs else None,
        (QK_L2NORM if qk_l2norm else 0) | (GATE_PER_CHANNEL if channel_gates else 0),
        _stream(dev))
    if rc != 0:
        raise DrError(rc, "dr_chunk_fwd")
    return (o, state_out, chunk_states) if want_cs else (o, state_out)


def recurrent_step(q, k, v, g, beta, state, scale: float = 1.0, out_dtype=torch.float32, o=None,
                   qk_l2norm: bool = False):
    """One decode step through ``dr_recurrent_step``; ``state`` is updated in place.

    q, k [B, Hqk, dk], v [B, Hv, dv] (bf16 or fp32); g (or None), beta [B, Hv] fp32;
    g may be [B, Hv, dk] (per key channel, as for ``chunk_fwd``); state [B, Hv, dk, dv] fp32.  ``qk_l2norm`` as for ``chunk_fwd``.  Returns o [B, Hv, dv] in
    ``out_dtype``.
    """
    if q.dtype not in _DTYPES or out_dtype not in _DTYPES:
        raise ValueError("q/k/v must be bf16 or fp32; out_dtype bf16 or fp32")
    dev = q.device
    for t, name, dt in ((q, "q", q.dtype), (k, "k", q.dtype), (v, "v", q.dtype),
                        (g, "g", torch.float32), (beta, "beta", torch.float32),
                        (state, "state", torch.float32)):
        _check(t, name, dt, dev)
    B, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if tuple(state.shape) != (B, Hv, dk, dv) or beta.shape != (B, Hv):
        raise ValueError("inconsistent shapes")
    channel_gates = g is not None and g.dim() == 3
    if g is not None and tuple(g.shape) not in ((B, Hv), (B, Hv, dk)):
        raise ValueError("g must be [B, Hv] or [B, Hv, dk]")
    if o is None:
        o = torch.empty((B, Hv, dv), dtype=out_dtype, device=dev)
    _check(o, "o", out_dtype, dev)
    rc = lib().dr_recurrent_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), B, Hqk, Hv, dk, dv,
        _DTYPES[q.dtype], float(scale), _ptr(o), _DTYPES[out_dtype],
        (QK_L2NORM if qk_l2norm else 0) | (GATE_PER_CHANNEL if channel_gates else 0),
        _stream(dev))
    if rc != 0:
        raise DrError(rc, "dr_recurrent_step")
    return o


def short_conv_silu(x, w, conv_state=None, cu_seqlens=None, out_dtype=None,
                    output_conv_state: bool = True):
    """Causal depthwise convolution + SiLU through ``dr_short_conv_silu``.

    x [B, T, H, d] (or [B, T, C]) bf16 or fp32; w [H, d, K] (or [C, K]) fp32, K <= 8;
    conv_state [N, H, d, K-1] fp32 or None (zero history); cu_seqlens int32 [N+1] or None.
    Returns (y like x in ``out_dtype`` (default x's dtype), conv_state_out or None).
    """
    if x.dtype not in _DTYPES:
        raise ValueError("x must be bf16 or fp32")
    out_dtype = x.dtype if out_dtype is None else out_dtype
    if out_dtype not in _DTYPES:
        raise ValueError("out_dtype must be bf16 or fp32")
    dev = x.device
    _check(x, "x", x.dtype, dev)
    _check(w, "w", torch.float32, dev)
    _check(conv_state, "conv_state", torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    B, T = x.shape[:2]
    C = math.prod(x.shape[2:])
    K = w.shape[-1]
    if w.numel() != C * K:
        raise ValueError("w must hold K taps per channel of x")
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if conv_state is not None and conv_state.numel() != N * C * (K - 1):
        raise ValueError("conv_state must be [N, channels, K-1]")
    y = torch.empty(x.shape, dtype=out_dtype, device=dev)
    st = (torch.empty((N,) + tuple(x.shape[2:]) + (K - 1,), dtype=torch.float32, device=dev)
          if output_conv_state else None)
    rc = lib().dr_short_conv_silu(
        _ptr(x), _DTYPES[x.dtype], _ptr(w), K, _ptr(conv_state), _ptr(st), _ptr(cu_seqlens),
        N, B, T, C, _ptr(y), _DTYPES[out_dtype], _stream(dev))
    if rc != 0:
        raise DrError(rc, "dr_short_conv_silu")
    return y, st


NORM_KINDS = {"rms": 0, "layer": 1}  # DR_NORM_RMS, DR_NORM_LAYER of include/dr.h


def norm_gate(o, weight, bias=None, z=None, kind: str = "rms", eps=None, out_dtype=None, y=None):
    """Per-(token, head) RMSNorm / LayerNorm over the last axis, then y * silu(z)
    through ``dr_norm_gate``.

    o [..., dv] bf16 or fp32 (dv <= 128); weight, bias [dv] fp32 (bias: LayerNorm only, or
    None); z like o (any of the two dtypes) or None.  eps defaults to 1e-6 (RMSNorm) or 1e-5
    (LayerNorm).  ``y`` may be ``o`` itself (in place) when the dtypes match; the output
    dtype is ``out_dtype``, else y's, else o's.
    """
    if o.dtype not in _DTYPES:
        raise ValueError("o must be bf16 or fp32")
    if out_dtype is None:
        out_dtype = o.dtype if y is None else y.dtype
    dev = o.device
    _check(o, "o", o.dtype, dev)
    _check(weight, "weight", torch.float32, dev)
    _check(bias, "bias", torch.float32, dev)
    if z is not None:
        _check(z, "z", z.dtype, dev)
        if z.dtype not in _DTYPES or z.shape != o.shape:
            raise ValueError("z must be bf16 or fp32 and shaped like o")
    dv = o.shape[-1]
    if weight.numel() != dv or (bias is not None and bias.numel() != dv):
        raise ValueError("weight / bias must have dv entries")
    if y is None:
        y = torch.empty(o.shape, dtype=out_dtype, device=dev)
    _check(y, "y", out_dtype, dev)
    if eps is None:
        eps = 1e-6 if kind == "rms" else 1e-5
    rc = lib().dr_norm_gate(
        _ptr(o), _DTYPES[o.dtype], _ptr(weight), _ptr(bias), _ptr(z),
        _DTYPES[z.dtype] if z is not None else 0, o.numel() // dv, dv, NORM_KINDS[kind],
        float(eps), _ptr(y), _DTYPES[out_dtype], _stream(dev))
    if rc != 0:
        raise DrError(rc, "dr_norm_gate")
    return y


KERNELS = {0: None, 1: "simt_f32", 2: "tc_bf16"}
QK_L2NORM = 1  # DR_QK_L2NORM of include/dr.h
GATE_PER_CHANNEL = 2  # DR_GATE_PER_CHANNEL of include/dr.h


def prefill_kernel(dtype, dk: int, dv: int, channel_gates: bool = False):
    """Name of the kernel dr_chunk_fwd picks for these inputs ('tc_bf16', 'simt_f32' or None)."""
    name = KERNELS[lib().dr_chunk_fwd_kernel(_DTYPES[dtype], dk, dv)]
    return "simt_f32" if (channel_gates and name is not None) else name


def device_status(device=None) -> int:
    """Synchronise and return (and clear) the library's device status code."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return int(lib().dr_get_device_status(_stream(dev)))
