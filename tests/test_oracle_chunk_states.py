"""Pins of the oracle's chunk-state output (the state at every chunk boundary).

The "linear_attention" page's recurrent route (LinearAttention) exposes the state
after every token; the oracle samples it after every ``chunk_len`` tokens of each
sequence and after the sequence's last token.  Checked against things other than the
token loop that writes them:
  CS1  exact rational brute force on every prefix (closed product of affine maps),
       varlen with an empty sequence and a ragged tail, dk != dv;
  CS2  the chunk (UT/WY) form's own end-of-chunk states, for several chunk lengths;
  CS3  a sequence's last row is its final state; chunk_len >= len gives one row per
       sequence; chunk_len = 1 gives the state after every token.
A boundary taken one token early or late, a row base that ignores an empty or ragged
sequence, or a transposed state fails one of these.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import brute, chunk_ref

from test_oracle_pins import _to_frac, rand_problem, rel


@pytest.mark.parametrize("chunk_len", [1, 2, 3, 7])
def test_cs1_exact_brute_force_on_prefixes(chunk_len):
    rng = np.random.default_rng(40 + chunk_len)
    cu = [0, 5, 5, 12]  # sequence 1 is empty
    T, dk, dv = cu[-1], 2, 3
    qf = [[_to_frac(x) for x in row] for row in rng.standard_normal((T, dk))]
    kf = [[_to_frac(x, 16) for x in row] for row in 0.5 * rng.standard_normal((T, dk))]
    vf = [[_to_frac(x) for x in row] for row in rng.standard_normal((T, dv))]
    af = [Fraction(int(rng.integers(1, 9)), 8) for _ in range(T)]
    bf = [Fraction(int(rng.integers(0, 33)), 16) for _ in range(T)]
    S0 = [[[_to_frac(x) for x in row] for row in rng.standard_normal((dv, dk))] for _ in range(3)]

    f = lambda m: np.array([[float(x) for x in row] for row in m])
    q = f(qf)[None, :, None, :]
    k = f(kf)[None, :, None, :]
    v = f(vf)[None, :, None, :]
    g = np.log(np.array([float(a) for a in af]))[None, :, None]
    beta = np.array([float(b) for b in bf])[None, :, None]
    s0 = np.stack([f(S).T for S in S0])[:, None]  # stored state is S^T
    _, _, cs = oracle.run(q, k, v, g, beta, s0, cu_seqlens=np.array(cu), chunk_len=chunk_len)

    bases, total = oracle.chunk_rows(cu, 1, T, chunk_len)
    assert cs.shape == (total, 1, dk, dv)
    for n in range(3):
        t0, t1 = cu[n], cu[n + 1]
        nrows = -(-(t1 - t0) // chunk_len)
        for j in range(nrows):
            e = t0 + min((j + 1) * chunk_len, t1 - t0)
            _, S_ex = brute.solve(qf[t0:e], kf[t0:e], vf[t0:e], af[t0:e], bf[t0:e], S0[n])
            assert rel(cs[bases[n] + j, 0], f(S_ex).T) < 1e-13, (n, j)
    assert total == -(-5 // chunk_len) + -(-7 // chunk_len)


@pytest.mark.parametrize("chunk_len", [4, 16, 64])
@pytest.mark.parametrize("varlen", [False, True])
def test_cs2_chunk_form_end_states(chunk_len, varlen):
    rng = np.random.default_rng(7 + chunk_len)
    if varlen:
        q, k, v, g, beta, _ = rand_problem(rng, B=1, T=150, dk=6, dv=4)
        cu = np.array([0, 37, 37, 101, 150])
        s0 = rng.standard_normal((4, 4, 6, 4)) * 0.5
    else:
        q, k, v, g, beta, s0 = rand_problem(rng, B=2, T=70, dk=6, dv=4)
        cu = None
    o, st, cs = oracle.run(q, k, v, g, beta, s0, cu_seqlens=cu, scale=0.5, chunk_len=chunk_len)
    oc, sc, csc = chunk_ref.run(q, k, v, g, beta, s0, cu_seqlens=cu, scale=0.5, chunk=chunk_len,
                                chunk_states=True)
    assert cs.shape == csc.shape
    assert rel(cs, csc) < 1e-11
    assert rel(o, oc) < 1e-11


def test_cs3_last_row_single_chunk_and_every_token():
    rng = np.random.default_rng(3)
    q, k, v, g, beta, _ = rand_problem(rng, B=1, T=40, Hqk=1, Hv=2, dk=4, dv=3)
    cu = np.array([0, 9, 9, 40])
    s0 = rng.standard_normal((3, 2, 4, 3))
    _, st, cs = oracle.run(q, k, v, g, beta, s0, cu_seqlens=cu, chunk_len=5)
    bases, total = oracle.chunk_rows(cu, 1, 40, 5)
    assert total == 2 + 0 + 7 and bases == [0, 2, 2]
    assert np.array_equal(cs[1], st[0]) and np.array_equal(cs[8], st[2])

    _, st, cs = oracle.run(q, k, v, g, beta, s0, cu_seqlens=cu, chunk_len=64)
    assert cs.shape[0] == 2 and np.array_equal(cs[0], st[0]) and np.array_equal(cs[1], st[2])

    # chunk_len = 1: row t of sequence 2 is the state after its first t + 1 tokens, which a
    # run over just those tokens ends in.
    _, _, cs = oracle.run(q, k, v, g, beta, s0, cu_seqlens=cu, chunk_len=1)
    assert cs.shape[0] == 40
    for t in (0, 13, 30):
        e = 9 + t + 1
        sl = lambda x: x[:, 9:e]
        _, s_pre = oracle.run(sl(q), sl(k), sl(v), sl(g), sl(beta), s0[2:3])
        assert np.array_equal(cs[9 + t], s_pre[0])


def test_cs_without_chunk_len_keeps_two_outputs():
    rng = np.random.default_rng(1)
    prob = rand_problem(rng, B=1, T=3, Hqk=1, Hv=1, dk=2, dv=2)
    assert len(oracle.run(*prob)) == 2
