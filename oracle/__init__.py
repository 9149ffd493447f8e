"""fp64 CPU oracle for the gated delta rule.

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``gated_delta_rule_59_b200``) never imports it, and
nothing here imports the product path.

Contents
  run(...)         token-by-token fp64 recurrence (C library ``liboracle.so``),
                   three independent update forms (see ``dr_oracle.c``); optional
                   q/k L2 normalisation first (``l2_normalize_rows``).
  chunk_ref        numpy fp64 chunk (UT/WY) form, used to pin the chunk algebra.
  brute            exact rational brute force on tiny inputs.
  layer            prologue and epilogue around the rule: short causal depthwise
                   convolution + SiLU, RMSNorm / LayerNorm + SiLU output gate.

Parity pins live in ``tests/test_oracle_*.py``.  Every function here is pinned:
the three forms against one another, against exact rational arithmetic
(``brute``), against closed forms (scalar recurrence, orthonormal-key recall,
Householder norm preservation) and invariants (beta = 0, g = 0, linearity).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        cmd = [
            "gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
            "-std=c11", "-Wall", "-o", _LIB_PATH, _SRC, "-lm",
        ]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        lib.oracle_run.argtypes = [
            dp, dp, dp, dp, dp, dp, ip,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int,
            dp, dp, ctypes.c_int, dp, ctypes.c_int,
        ]
        lib.oracle_run.restype = ctypes.c_int
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor on the CPU
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, typ=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(typ))


def l2_normalize_rows(x):
    """Each row (last axis) divided by its Euclidean norm, in fp64; an all-zero row stays zero.

    "DeltaNet Attention" (class docstring) and "DeltaNet" (section "The Delta Rule") state that
    queries and keys are L2-normalised before the rule; the "linear_attention" page draws it as
    the ``qk_l2norm`` block in front of ``delta_rule``.  No epsilon is given: the plain quotient
    is taken, with the zero row mapped to zero.
    """
    x = _f64(x)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return np.where(n > 0.0, x / np.where(n > 0.0, n, 1.0), 0.0)


def chunk_rows(cu_seqlens, B: int, T: int, chunk_len: int):
    """First chunk-state row of every sequence and the total row count.

    Sequence n owns ceil(len_n / chunk_len) rows, in sequence order; a sequence of length
    zero owns none.  Returns (bases [N] as a list of ints, total).
    """
    if cu_seqlens is None:
        lens = [T] * B
    else:
        cu = [int(x) for x in np.asarray(cu_seqlens)]
        lens = [cu[n + 1] - cu[n] for n in range(len(cu) - 1)]
    bases, tot = [], 0
    for ln in lens:
        bases.append(tot)
        tot += -(-ln // chunk_len)
    return bases, tot


def run(q, k, v, g, beta, state_in=None, cu_seqlens=None, scale: float = 1.0,
        form: int = 2, threads: int = 0, qk_l2norm: bool = False, chunk_len: int = 0):
    """Token-by-token fp64 recurrence.

    q, k: [B, T, Hqk, dk]; v: [B, T, Hv, dv]; g, beta: [B, T, Hv] (g may be None);
    g may also be [B, T, Hv, dk]: one log decay per key channel (the "linear_attention"
    page's ChannelGates), which scales row i of the stored state by exp(g[..., i]);
    state_in: [N, Hv, dk, dv] or None (zeros); cu_seqlens: int [N+1] or None.
    ``qk_l2norm``: q and k rows are L2-normalised first (``l2_normalize_rows``).
    Returns (o [B, T, Hv, dv], state_out [N, Hv, dk, dv]) as float64 numpy arrays.
    With ``chunk_len`` > 0 a third array is returned: the stored state after every
    ``chunk_len`` tokens of each sequence and after its last token,
    [sum_n ceil(len_n / chunk_len), Hv, dk, dv], rows ordered as ``chunk_rows`` gives.
    These sample, at chunk boundaries, the state after every token that the
    "linear_attention" page (LinearAttention, its recurrent route) exposes for tracing.
    """
    lib = _load()
    q, k, v, g, beta, state_in = (_f64(a) for a in (q, k, v, g, beta, state_in))
    if qk_l2norm:
        q, k = np.ascontiguousarray(l2_normalize_rows(q)), np.ascontiguousarray(l2_normalize_rows(k))
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    assert k.shape == q.shape and v.shape[:2] == (B, T) and beta.shape == (B, T, Hv)
    channel_gates = g is not None and g.ndim == 4
    if g is not None:
        assert g.shape == ((B, T, Hv, dk) if channel_gates else (B, T, Hv)), g.shape
    cu = None
    if cu_seqlens is not None:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        N = cu.shape[0] - 1
    else:
        N = B
    if state_in is not None:
        assert state_in.shape == (N, Hv, dk, dv), state_in.shape
    o = np.zeros((B, T, Hv, dv), dtype=np.float64)
    st = np.zeros((N, Hv, dk, dv), dtype=np.float64)
    cs = None
    if chunk_len > 0:
        cs = np.zeros((chunk_rows(cu, B, T, chunk_len)[1], Hv, dk, dv), dtype=np.float64)
    rc = lib.oracle_run(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in),
        _ptr(cu, ctypes.c_int32), N, B, T, Hqk, Hv, dk, dv, float(scale), int(form),
        int(threads), _ptr(o), _ptr(st), int(chunk_len), _ptr(cs), int(channel_gates),
    )
    if rc != 0:
        raise ValueError(f"oracle_run failed with code {rc}")
    return (o, st) if cs is None else (o, st, cs)


def step(q, k, v, g, beta, state, scale: float = 1.0, form: int = 2, threads: int = 0,
         qk_l2norm: bool = False):
    """One decode step (T = 1) for every (batch, v-head).

    q, k: [B, Hqk, dk]; v: [B, Hv, dv]; g, beta: [B, Hv] (g may be [B, Hv, dk]: per key
    channel); state: [B, Hv, dk, dv].
    Returns (o [B, Hv, dv], new_state [B, Hv, dk, dv]); ``state`` is not modified.
    """
    q, k, v, beta, state = (_f64(a) for a in (q, k, v, beta, state))
    g = _f64(g)
    o, st = run(q[:, None], k[:, None], v[:, None], None if g is None else g[:, None],
                beta[:, None], state, None, scale, form, threads, qk_l2norm)
    return o[:, 0], st
