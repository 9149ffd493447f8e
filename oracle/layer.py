"""fp64 prologue and epilogue around the delta rule: short convolution + SiLU before it,
normalisation + SiLU output gate after it.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages draw around the rule:
  - "DeltaNet" (study notes, the layer diagram): q/k and v each pass a projection, a
    convolution ("Conv*", depthwise, generalising the shift SSM) and a SiLU; q and k
    are then L2-normalised; the rule's output goes through an RMSNorm and the output
    projection.
  - "DeltaNet Attention" (class docstring and attributes): the readout is normalised by
    ``norm`` (an ``nn.LayerNorm``) and then modulated channel-wise by a SiLU-gated
    output projection (``g_proj``).
The projections carry weights and are not part of this path: the prologue starts from
the projected q/k/v, and the gate from the projected gate input z.

Readings where the pages are silent:
  - the convolution is causal, one filter of K taps per channel (depthwise), no bias;
    K is a parameter (4 by default).  Tap K-1 weighs the current token, tap j the token
    K-1-j steps back.  Before a sequence's first token the history is zero, or the
    ``conv_state`` of a previous call: the last K-1 inputs, oldest first.  Sequences of a
    varlen batch never see one another.
  - the normalisation acts per token and head over the d_v outputs, with one weight
    vector of d_v entries shared by all heads; RMSNorm eps = 1e-6, LayerNorm eps = 1e-5
    (the ``nn.LayerNorm`` default) with biased variance and a bias vector.
  - the gate multiplies the normalised readout by silu(z), z [B, T, Hv, d_v].
"""
from __future__ import annotations

import numpy as np

from . import _f64  # float64 numpy view of a numpy array or a torch tensor of any dtype


def silu(x):
    """x sigmoid(x), evaluated without overflow for large negative x."""
    x = _f64(x)
    return np.where(x >= 0, x / (1.0 + np.exp(-np.abs(x))),
                    x * np.exp(-np.abs(x)) / (1.0 + np.exp(-np.abs(x))))


def _sequences(cu_seqlens, B, T):
    if cu_seqlens is None:
        return [(b, 0, T) for b in range(B)]
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    return [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]


def short_conv_silu(x, w, conv_state=None, cu_seqlens=None):
    """Causal depthwise convolution, then SiLU.

    x [B, T, H, d] (projected q, k or v); w [H, d, K]; conv_state [N, H, d, K-1] or None
    (zero history).  Returns (y [B, T, H, d], conv_state_out [N, H, d, K-1]): y_t[c] =
    silu(sum_j w[c, j] x_{t-K+1+j}[c]), and conv_state_out holds the last K-1 inputs of
    each sequence (history included when the sequence is shorter than K-1).
    """
    x, w = _f64(x), _f64(w)
    B, T, H, d = x.shape
    K = w.shape[-1]
    assert w.shape == (H, d, K)
    seqs = _sequences(cu_seqlens, B, T)
    y = np.zeros_like(x)
    st_out = np.zeros((len(seqs), H, d, K - 1))
    for n, (b, t0, t1) in enumerate(seqs):
        hist = (np.zeros((K - 1, H, d)) if conv_state is None
                else np.moveaxis(_f64(conv_state[n]), -1, 0))
        xp = np.concatenate([hist, x[b, t0:t1]], axis=0)  # [K-1 + L, H, d]
        for t in range(t1 - t0):
            acc = np.zeros((H, d))
            for j in range(K):
                acc += w[:, :, j] * xp[t + j]
            y[b, t0 + t] = silu(acc)
        if K > 1:
            st_out[n] = np.moveaxis(xp[-(K - 1):], 0, -1)
    return y, st_out


def norm_gate(o, weight, bias=None, z=None, kind="rms", eps=None):
    """Per-(token, head) normalisation over d_v, then the optional SiLU output gate.

    o [B, T, Hv, dv]; weight [dv]; bias [dv] or None (LayerNorm only); z like o or None.
    kind "rms":   y = o / sqrt(mean(o^2) + eps) * weight                (eps 1e-6)
    kind "layer": y = (o - mean(o)) / sqrt(var(o) + eps) * weight + bias  (eps 1e-5)
    then y * silu(z) when z is given.
    """
    o, weight = _f64(o), _f64(weight)
    if kind == "rms":
        e = 1e-6 if eps is None else eps
        y = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + e) * weight
    elif kind == "layer":
        e = 1e-5 if eps is None else eps
        mu = np.mean(o, axis=-1, keepdims=True)
        var = np.mean((o - mu) ** 2, axis=-1, keepdims=True)
        y = (o - mu) / np.sqrt(var + e) * weight
        if bias is not None:
            y = y + _f64(bias)
    else:
        raise ValueError(kind)
    if z is not None:
        y = y * silu(z)
    return y


def mixer(qx, kx, vx, wq, wk, wv, g, beta, state_in=None, cu_seqlens=None, scale=1.0,
          conv_states=(None, None, None), norm_weight=None, norm_bias=None, z=None,
          norm_kind="rms"):
    """Projected inputs -> conv + SiLU -> L2 norm (q, k) -> delta rule -> norm -> gate.

    Returns (out [B, T, Hv, dv], state_out [N, Hv, dk, dv], (q, k, v conv states)).
    """
    from . import run

    q, cq = short_conv_silu(qx, wq, conv_states[0], cu_seqlens)
    k, ck = short_conv_silu(kx, wk, conv_states[1], cu_seqlens)
    v, cv = short_conv_silu(vx, wv, conv_states[2], cu_seqlens)
    o, st = run(q, k, v, g, beta, state_in, cu_seqlens, scale=scale, qk_l2norm=True)
    dv = o.shape[-1]
    wn = np.ones(dv) if norm_weight is None else norm_weight
    return norm_gate(o, wn, norm_bias, z, norm_kind), st, (cq, ck, cv)
