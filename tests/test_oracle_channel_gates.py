"""Pins of the oracle's per-key-channel gates (the "linear_attention" page's ChannelGates).

g [B, T, Hv, dk] holds one log kept-fraction per key channel; the state's key row i
decays by exp(g_t[i]) before the delta write.  Checked against things other than the
token loop:
  CG1  equal entries across channels reproduce the scalar gate;
  CG2  exact rational brute force with a diagonal decay (closed product of affine maps),
       all three update forms, dk != dv;
  CG3  the chunk (UT/WY) form with per-channel decay, several chunk lengths, varlen;
  CG4  beta = 0: the state is diag(exp(sum g)) H0 and o_t reads diag(exp(b_t)) H0;
  CG5  key rows outside the keys' support only decay, row by row, whatever else happens.
A decay applied to value columns instead of key rows, a decay after the write, or a
dropped channel fails at least one of these.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import brute, chunk_ref

from test_oracle_pins import _to_frac, rand_problem, rel


def channel_g(rng, B, T, Hv, dk, spread=1.0):
    return np.log(rng.uniform(0.2, 1.0, (B, T, Hv, dk))) * spread


@pytest.mark.parametrize("seed", range(3))
def test_cg1_equal_channels_are_the_scalar_gate(seed):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, s0 = rand_problem(rng, B=2, T=20, dk=5, dv=3)
    gc = np.repeat(g[..., None], 5, axis=-1)
    for form in (1, 2, 3):
        o1, s1 = oracle.run(q, k, v, g, beta, s0, form=form)
        o2, s2 = oracle.run(q, k, v, gc, beta, s0, form=form)
        assert rel(o2, o1) < 1e-14 and rel(s2, s1) < 1e-14


@pytest.mark.parametrize("seed", range(3))
@pytest.mark.parametrize("form", [1, 2, 3])
def test_cg2_exact_rational_brute_force(seed, form):
    rng = np.random.default_rng(200 + seed)
    T, dk, dv = 5, 3, 2
    qf = [[_to_frac(x) for x in row] for row in rng.standard_normal((T, dk))]
    kf = [[_to_frac(x, 16) for x in row] for row in 0.5 * rng.standard_normal((T, dk))]
    vf = [[_to_frac(x) for x in row] for row in rng.standard_normal((T, dv))]
    af = [[Fraction(int(rng.integers(1, 9)), 8) for _ in range(dk)] for _ in range(T)]
    bf = [Fraction(int(rng.integers(0, 33)), 16) for _ in range(T)]
    S0 = [[_to_frac(x) for x in row] for row in rng.standard_normal((dv, dk))]
    o_ex, S_ex = brute.solve(qf, kf, vf, af, bf, S0)

    f = lambda m: np.array([[float(x) for x in row] for row in m])
    q = f(qf)[None, :, None, :]
    k = f(kf)[None, :, None, :]
    v = f(vf)[None, :, None, :]
    g = np.log(f(af))[None, :, None, :]
    beta = np.array([float(b) for b in bf])[None, :, None]
    o, st = oracle.run(q, k, v, g, beta, f(S0).T[None, None], form=form)
    assert rel(o[0, :, 0, :], f(o_ex)) < 1e-13
    assert rel(st[0, 0], f(S_ex).T) < 1e-13


@pytest.mark.parametrize("C", [1, 5, 16, 64])
def test_cg3_chunk_form(C):
    rng = np.random.default_rng(30 + C)
    q, k, v, _, beta, s0 = rand_problem(rng, B=2, T=90, dk=6, dv=4)
    g = channel_g(rng, 2, 90, 4, 6, spread=2.0)
    o, s = oracle.run(q, k, v, g, beta, s0, scale=0.5)
    oc, sc = chunk_ref.run(q, k, v, g, beta, s0, scale=0.5, chunk=C)
    assert rel(oc, o) < 1e-11 and rel(sc, s) < 1e-11


def test_cg3_chunk_form_varlen_with_chunk_states():
    rng = np.random.default_rng(5)
    q, k, v, _, beta, _ = rand_problem(rng, B=1, T=150, dk=6, dv=4)
    g = channel_g(rng, 1, 150, 4, 6)
    cu = np.array([0, 37, 37, 101, 150])
    s0 = rng.standard_normal((4, 4, 6, 4)) * 0.5
    o, s, cs = oracle.run(q, k, v, g, beta, s0, cu_seqlens=cu, chunk_len=16)
    oc, sc, csc = chunk_ref.run(q, k, v, g, beta, s0, cu_seqlens=cu, chunk=16, chunk_states=True)
    assert rel(oc, o) < 1e-11 and rel(sc, s) < 1e-11 and rel(csc, cs) < 1e-11


def test_cg4_beta_zero_is_pure_channel_decay():
    rng = np.random.default_rng(8)
    q, k, v, _, _, s0 = rand_problem(rng, B=1, T=12, Hqk=1, Hv=2, dk=4, dv=3)
    g = channel_g(rng, 1, 12, 2, 4)
    beta = np.zeros((1, 12, 2))
    o, s = oracle.run(q, k, v, g, beta, s0)
    b = np.cumsum(g[0], axis=0)  # [T, Hv, dk]
    for h in range(2):
        assert rel(s[0, h], np.exp(b[-1, h])[:, None] * s0[0, h]) < 1e-13
        for t in (0, 5, 11):
            Ht = np.exp(b[t, h])[:, None] * s0[0, h]
            assert rel(o[0, t, h], Ht.T @ q[0, t, 0]) < 1e-13


def test_cg5_rows_outside_the_key_support_only_decay():
    rng = np.random.default_rng(9)
    q, k, v, _, beta, s0 = rand_problem(rng, B=1, T=15, Hqk=1, Hv=1, dk=6, dv=3)
    k[..., 3:] = 0.0  # keys live in channels 0..2
    g = channel_g(rng, 1, 15, 1, 6, spread=1.5)
    _, s = oracle.run(q, k, v, g, beta, s0)
    decay = np.exp(np.sum(g[0, :, 0, 3:], axis=0))
    assert rel(s[0, 0, 3:], decay[:, None] * s0[0, 0, 3:]) < 1e-13
    # and the channels with keys did take writes
    assert np.max(np.abs(s[0, 0, :3] - np.exp(np.sum(g[0, :, 0, :3], axis=0))[:, None]
                         * s0[0, 0, :3])) > 1e-3


def test_golden_exact_fixture_with_chunk_states():
    """Exact rational values written by tests/golden/make_golden.py (brute force only)."""
    import json
    import os

    path = os.path.join(os.path.dirname(__file__), "golden", "brute_channel_gates.json")
    with open(path) as fh:
        fx = json.load(fh)
    F = lambda x: float(Fraction(x))
    arr = lambda m: np.array([[F(x) for x in row] for row in m])
    q, k, v, S0 = arr(fx["q"]), arr(fx["k"]), arr(fx["v"]), arr(fx["S0"])
    g = np.log(arr(fx["alpha"]))
    beta = np.array([F(b) for b in fx["beta"]])
    o, st, cs = oracle.run(q[None, :, None], k[None, :, None], v[None, :, None],
                           g[None, :, None, :], beta[None, :, None], S0.T[None, None],
                           chunk_len=2)
    assert rel(o[0, :, 0], arr(fx["o"])) < 1e-13
    assert rel(st[0, 0], arr(fx["S_T"]).T) < 1e-13
    for j, S in enumerate(fx["S_after"]):
        assert rel(cs[j, 0], arr(S).T) < 1e-13

