"""Pins of the oracle's prologue and epilogue around the rule (``oracle/layer.py``).

  L1  the convolution against numpy's own convolution, channel by channel;
  L2  causality: a unit impulse returns the taps, in order, from its token onward;
  L3  a sequence split in two with the conv state carried over equals the unsplit one;
      a varlen batch equals separate calls (no history crosses a boundary);
  L4  one tap of weight 1 is SiLU alone; SiLU against torch's;
  L5  RMSNorm and LayerNorm against torch's functional forms, the gate against torch's
      SiLU; RMSNorm with eps = 0 has unit RMS and ignores a positive rescaling;
  L6  the composed mixer equals its steps and reads the L2-normalised q, k.
A tap order reversed, a history shifted by one, a norm over the wrong axis or a gate
applied before the norm fails one of these.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import layer


def rel(a, b):
    return np.max(np.abs(np.asarray(a) - np.asarray(b))) / max(np.max(np.abs(b)), 1e-300)


def _silu_torch(x):
    return torch.nn.functional.silu(torch.as_tensor(x, dtype=torch.float64)).numpy()


@pytest.mark.parametrize("K", [1, 2, 4])
def test_l1_against_numpy_convolution(K):
    rng = np.random.default_rng(K)
    B, T, H, d = 2, 13, 2, 3
    x = rng.standard_normal((B, T, H, d))
    w = rng.standard_normal((H, d, K))
    y, _ = layer.short_conv_silu(x, w)
    for b in range(B):
        for h in range(H):
            for c in range(d):
                # numpy convolves with the flipped kernel: tap K-1 meets the current token
                pre = np.convolve(x[b, :, h, c], w[h, c, ::-1])[:T]
                assert rel(y[b, :, h, c], _silu_torch(pre)) < 1e-14


def test_l2_impulse_response_is_causal():
    K, T = 4, 10
    w = np.arange(1.0, K + 1.0).reshape(1, 1, K)  # taps 1, 2, 3, 4
    x = np.zeros((1, T, 1, 1))
    x[0, 3] = 1.0
    y, _ = layer.short_conv_silu(x, w)
    pre = np.zeros(T)
    pre[3:3 + K] = w[0, 0, ::-1]  # the current token meets tap K-1, the next one tap K-2 ...
    assert rel(y[0, :, 0, 0], _silu_torch(pre)) < 1e-15
    assert np.all(y[0, :3] == 0.0)


@pytest.mark.parametrize("split", [1, 2, 5, 11])
def test_l3_state_carry_and_varlen(split):
    rng = np.random.default_rng(10 + split)
    T, H, d, K = 12, 2, 3, 4
    x = rng.standard_normal((1, T, H, d))
    w = rng.standard_normal((H, d, K))
    s0 = rng.standard_normal((1, H, d, K - 1))
    y, s = layer.short_conv_silu(x, w, s0)
    y1, s1 = layer.short_conv_silu(x[:, :split], w, s0)
    y2, s2 = layer.short_conv_silu(x[:, split:], w, s1)
    assert rel(np.concatenate([y1, y2], axis=1), y) < 1e-15 and rel(s2, s) < 1e-15
    # varlen: three sequences packed (one empty) equal three separate calls
    cu = np.array([0, split, split, T])
    S0 = rng.standard_normal((3, H, d, K - 1))
    yv, sv = layer.short_conv_silu(x, w, S0, cu)
    for n in range(3):
        a, b = cu[n], cu[n + 1]
        yn, sn = layer.short_conv_silu(x[:, a:b], w, S0[n:n + 1])
        assert rel(yv[:, a:b], yn) < 1e-15 if b > a else True
        assert rel(sv[n], sn[0]) < 1e-15


def test_l3_short_sequence_keeps_history_in_state():
    w = np.ones((1, 1, 4))
    s0 = np.array([1.0, 2.0, 3.0]).reshape(1, 1, 1, 3)
    x = np.array([7.0]).reshape(1, 1, 1, 1)
    y, s = layer.short_conv_silu(x, w, s0)
    assert np.array_equal(s[0, 0, 0], [2.0, 3.0, 7.0])
    assert rel(y[0, 0, 0, 0], _silu_torch(13.0)) < 1e-15


def test_l4_single_tap_is_silu():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 9, 3, 5)) * 30.0  # includes large negative values
    y, s = layer.short_conv_silu(x, np.ones((3, 5, 1)))
    assert rel(y, _silu_torch(x)) < 1e-14 and s.shape == (2, 3, 5, 0)


@pytest.mark.parametrize("kind", ["rms", "layer"])
def test_l5_norms_and_gate_against_torch(kind):
    rng = np.random.default_rng(5)
    o = rng.standard_normal((2, 7, 3, 16)) * 3.0
    wt = rng.uniform(0.5, 1.5, 16)
    bs = rng.standard_normal(16)
    z = rng.standard_normal(o.shape) * 2.0
    T = lambda a: torch.as_tensor(a, dtype=torch.float64)
    if kind == "rms":
        ref = torch.nn.functional.rms_norm(T(o), (16,), T(wt), eps=1e-6).numpy()
        got = layer.norm_gate(o, wt, kind="rms")
    else:
        ref = torch.nn.functional.layer_norm(T(o), (16,), T(wt), T(bs), eps=1e-5).numpy()
        got = layer.norm_gate(o, wt, bs, kind="layer")
    assert rel(got, ref) < 1e-13
    gated = layer.norm_gate(o, wt, bs if kind == "layer" else None, z, kind=kind)
    assert rel(gated, ref * _silu_torch(z)) < 1e-13


def test_l5_rms_invariants():
    rng = np.random.default_rng(6)
    o = rng.standard_normal((1, 5, 2, 32))
    y = layer.norm_gate(o, np.ones(32), kind="rms", eps=0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-14, rtol=0)
    assert rel(layer.norm_gate(7.5 * o, np.ones(32), kind="rms", eps=0.0), y) < 1e-14


def test_l6_mixer_composes_its_steps():
    rng = np.random.default_rng(7)
    B, T, Hqk, Hv, d, K = 1, 20, 1, 2, 8, 4
    qx, kx = rng.standard_normal((2, B, T, Hqk, d))
    vx = rng.standard_normal((B, T, Hv, d))
    wq, wk = rng.standard_normal((2, Hqk, d, K)) * 0.5
    wv = rng.standard_normal((Hv, d, K)) * 0.5
    g = np.log(rng.uniform(0.5, 1.0, (B, T, Hv)))
    beta = rng.uniform(0, 1, (B, T, Hv))
    z = rng.standard_normal((B, T, Hv, d))
    out, st, convs = layer.mixer(qx, kx, vx, wq, wk, wv, g, beta, scale=d ** -0.5, z=z)
    q, _ = layer.short_conv_silu(qx, wq)
    k, _ = layer.short_conv_silu(kx, wk)
    v, _ = layer.short_conv_silu(vx, wv)
    qn, kn = oracle.l2_normalize_rows(q), oracle.l2_normalize_rows(k)
    o, st2 = oracle.run(qn, kn, v, g, beta, scale=d ** -0.5)
    assert rel(out, layer.norm_gate(o, np.ones(d), z=z)) < 1e-13 and rel(st, st2) < 1e-13
    assert all(c.shape[-1] == K - 1 for c in convs)
