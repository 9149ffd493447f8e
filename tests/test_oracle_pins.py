"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself:
  P1  the three update forms of the pages agree (projection form of "DeltaNet
      Attention"; error-correction/SGD and retrieve-and-replace forms of
      "DeltaNet", section "The Delta Rule");
  P5  exact rational brute force (closed product of affine maps);
  I1  beta = 0 leaves the state unchanged up to the decay;
  I2  beta = 1 with orthonormal keys gives exact recall (the MQAR mechanism of
      the "DeltaNet Attention" class docstring);
  I3  g = 0 reduces the gated rule of "linear_attention" to plain DeltaNet;
  I4  beta = 2 (the allow-negative-eigenvalue range) is a Householder
      reflection: norm preserving; beta in [0, 1] is non-expansive;
  I5  linearity in (initial state, values);
  I6  d = 1 closed form of a first-order linear recurrence.
A mistake in any single place (dropped decay, wrong sign, state transposed,
read before write, wrong head mapping) fails at least one of these.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import brute


def rand_problem(rng, B=2, T=11, Hqk=2, Hv=4, dk=5, dv=3, gated=True, beta_max=2.0,
                 state=True, normalise=False):
    q = rng.standard_normal((B, T, Hqk, dk))
    k = rng.standard_normal((B, T, Hqk, dk)) * 0.6
    if normalise:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, Hv, dv))
    g = np.log(rng.uniform(0.3, 1.0, (B, T, Hv))) if gated else None
    beta = rng.uniform(0.0, beta_max, (B, T, Hv))
    s0 = rng.standard_normal((B, Hv, dk, dv)) * 0.5 if state else None
    return q, k, v, g, beta, s0


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("gated", [False, True])
def test_p1_three_forms_agree(seed, gated):
    rng = np.random.default_rng(seed)
    prob = rand_problem(rng, gated=gated)
    o1, s1 = oracle.run(*prob, form=1)
    o2, s2 = oracle.run(*prob, form=2)
    o3, s3 = oracle.run(*prob, form=3)
    assert rel(o1, o2) < 1e-12 and rel(o3, o2) < 1e-12
    assert rel(s1, s2) < 1e-12 and rel(s3, s2) < 1e-12


def _to_frac(x, denom=64):
    return Fraction(int(round(float(x) * denom)), denom)


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("form", [1, 2, 3])
def test_p5_exact_rational_brute_force(seed, form):
    rng = np.random.default_rng(100 + seed)
    T, dk, dv = 5, 3, 2
    # dyadic rationals: exactly representable in float64
    qf = [[_to_frac(x) for x in row] for row in rng.standard_normal((T, dk))]
    kf = [[_to_frac(x, 16) for x in row] for row in 0.5 * rng.standard_normal((T, dk))]
    vf = [[_to_frac(x) for x in row] for row in rng.standard_normal((T, dv))]
    af = [Fraction(int(rng.integers(1, 9)), 8) for _ in range(T)]  # alpha in (0, 1]
    bf = [Fraction(int(rng.integers(0, 33)), 16) for _ in range(T)]  # beta in [0, 2]
    S0 = [[_to_frac(x) for x in row] for row in rng.standard_normal((dv, dk))]
    o_ex, S_ex = brute.solve(qf, kf, vf, af, bf, S0)

    f = lambda m: np.array([[float(x) for x in row] for row in m])
    q = f(qf)[None, :, None, :]
    k = f(kf)[None, :, None, :]
    v = f(vf)[None, :, None, :]
    g = np.log(np.array([float(a) for a in af]))[None, :, None]
    beta = np.array([float(b) for b in bf])[None, :, None]
    s0 = f(S0).T[None, None]  # stored state is S^T
    o, st = oracle.run(q, k, v, g, beta, s0, form=form)
    assert rel(o[0, :, 0, :], f(o_ex)) < 1e-13
    assert rel(st[0, 0], f(S_ex).T) < 1e-13


def test_golden_exact_fixture():
    """Exact rational values written by tests/golden/make_golden.py (brute force only)."""
    import json
    import os

    path = os.path.join(os.path.dirname(__file__), "golden", "brute_tiny.json")
    with open(path) as fh:
        fx = json.load(fh)
    F = lambda s: float(Fraction(s))
    arr = lambda m: np.array([[F(x) for x in row] for row in m])
    q, k, v, S0 = arr(fx["q"]), arr(fx["k"]), arr(fx["v"]), arr(fx["S0"])
    alpha = np.array([F(a) for a in fx["alpha"]])
    beta = np.array([F(b) for b in fx["beta"]])
    o, st = oracle.run(q[None, :, None], k[None, :, None], v[None, :, None],
                       np.log(alpha)[None, :, None], beta[None, :, None], S0.T[None, None])
    assert rel(o[0, :, 0], arr(fx["o"])) < 1e-13
    assert rel(st[0, 0], arr(fx["S_T"]).T) < 1e-13


@pytest.mark.parametrize("seed", range(3))
def test_i1_beta_zero_is_pure_decay(seed):
    rng = np.random.default_rng(200 + seed)
    q, k, v, g, beta, s0 = rand_problem(rng)
    beta = np.zeros_like(beta)
    o, st = oracle.run(q, k, v, g, beta, s0)
    b = np.cumsum(g, axis=1)  # [B, T, Hv]
    Hqk, Hv = q.shape[2], v.shape[2]
    grp = Hv // Hqk
    for bb in range(q.shape[0]):
        for h in range(Hv):
            np.testing.assert_allclose(st[bb, h], np.exp(b[bb, -1, h]) * s0[bb, h], rtol=1e-12)
            for t in range(q.shape[1]):
                exp_o = np.exp(b[bb, t, h]) * (s0[bb, h].T @ q[bb, t, h // grp])
                np.testing.assert_allclose(o[bb, t, h], exp_o, rtol=1e-11, atol=1e-14)


@pytest.mark.parametrize("n_keys", [1, 3, 6])
@pytest.mark.parametrize("gated", [False, True])
def test_i2_orthonormal_keys_exact_recall(n_keys, gated):
    rng = np.random.default_rng(300 + n_keys)
    dk, dv = 6, 4
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm.T[:n_keys]  # orthonormal rows
    vals = rng.standard_normal((n_keys, dv))
    k = keys[None, :, None, :]
    q = k.copy()
    v = vals[None, :, None, :]
    beta = np.ones((1, n_keys, 1))
    alpha = rng.uniform(0.5, 1.0, n_keys) if gated else np.ones(n_keys)
    g = np.log(alpha)[None, :, None]
    s0 = rng.standard_normal((1, 1, dk, dv))
    _, st = oracle.run(q, k, v, g, beta, s0)
    S = st[0, 0].T  # math state, d_v x d_k
    for i in range(n_keys):
        decay = np.prod(alpha[i + 1:])
        np.testing.assert_allclose(S @ keys[i], decay * vals[i], atol=1e-12)
    if n_keys == dk and not gated:
        # the initial state is fully overwritten: S = sum_i v_i k_i^T
        np.testing.assert_allclose(S, vals.T @ keys, atol=1e-12)


def test_i3_zero_gate_is_plain_deltanet():
    rng = np.random.default_rng(400)
    q, k, v, _, beta, s0 = rand_problem(rng, gated=False)
    o_none, s_none = oracle.run(q, k, v, None, beta, s0)
    zeros = np.zeros(beta.shape)
    o_zero, s_zero = oracle.run(q, k, v, zeros, beta, s0)
    assert np.array_equal(o_none, o_zero) and np.array_equal(s_none, s_zero)
    # and the ungated projection form S (I - b k k^T) + b v k^T written out here
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    for bb in range(B):
        for h in range(Hv):
            S = s0[bb, h].T.copy()
            for t in range(T):
                kt = k[bb, t, h // (Hv // Hqk)]
                S = S @ (np.eye(dk) - beta[bb, t, h] * np.outer(kt, kt)) + beta[bb, t, h] * np.outer(v[bb, t, h], kt)
            np.testing.assert_allclose(s_none[bb, h], S.T, rtol=1e-11, atol=1e-13)


def test_i4_householder_norm_preserving_and_contraction():
    rng = np.random.default_rng(500)
    T, dk, dv = 12, 5, 4
    k = rng.standard_normal((1, T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q = rng.standard_normal((1, T, 1, dk))
    v = np.zeros((1, T, 1, dv))
    s0 = rng.standard_normal((1, 1, dk, dv))
    _, st = oracle.run(q, k, v, None, 2.0 * np.ones((1, T, 1)), s0)
    assert abs(np.linalg.norm(st) - np.linalg.norm(s0)) < 1e-12 * np.linalg.norm(s0)
    prev = np.linalg.norm(s0[0, 0], 2)
    bt = rng.uniform(0, 1, (1, T, 1))
    for t in range(1, T + 1):
        _, st_t = oracle.run(q[:, :t], k[:, :t], v[:, :t], None, bt[:, :t], s0)
        cur = np.linalg.norm(st_t[0, 0], 2)
        assert cur <= prev + 1e-12
        prev = cur


def test_i5_linearity_in_state_and_values():
    rng = np.random.default_rng(600)
    q, k, v, g, beta, s0 = rand_problem(rng)
    v2 = rng.standard_normal(v.shape)
    s02 = rng.standard_normal(s0.shape)
    c = -1.7
    oa, sa = oracle.run(q, k, v, g, beta, s0)
    ob, sb = oracle.run(q, k, v2, g, beta, s02)
    oc, sc = oracle.run(q, k, v + c * v2, g, beta, s0 + c * s02)
    np.testing.assert_allclose(oc, oa + c * ob, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(sc, sa + c * sb, rtol=1e-10, atol=1e-12)


def test_i6_scalar_closed_form():
    rng = np.random.default_rng(700)
    T = 40
    q = rng.standard_normal(T)
    k = rng.standard_normal(T)
    v = rng.standard_normal(T)
    g = np.log(rng.uniform(0.2, 1.0, T))
    beta = rng.uniform(0, 2, T)
    s0 = 0.7
    a = np.exp(g) * (1 - beta * k * k)  # s_t = a_t s_{t-1} + c_t
    c = beta * v * k
    # closed form: s_t = (prod_{j<=t} a_j) s0 + sum_{i<=t} c_i prod_{i<j<=t} a_j
    s = np.empty(T)
    for t in range(T):
        tot = np.prod(a[: t + 1]) * s0
        for i in range(t + 1):
            tot += c[i] * np.prod(a[i + 1: t + 1])
        s[t] = tot
    o, st = oracle.run(q[None, :, None, None], k[None, :, None, None], v[None, :, None, None],
                       g[None, :, None], beta[None, :, None], np.array([[[[s0]]]]))
    np.testing.assert_allclose(o[0, :, 0, 0], s * q, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(st[0, 0, 0, 0], s[-1], rtol=1e-11)


def test_scale_multiplies_query():
    rng = np.random.default_rng(800)
    prob = rand_problem(rng)
    o1, s1 = oracle.run(*prob, scale=1.0)
    o2, s2 = oracle.run(*prob, scale=0.25)
    np.testing.assert_allclose(o2, 0.25 * o1, rtol=1e-13, atol=1e-15)
    assert np.array_equal(s1, s2)
