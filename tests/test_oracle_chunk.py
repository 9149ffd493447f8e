"""P6: the chunk (UT/WY) form equals the token oracle for any chunk size.

The chunk form is the algebra every prefill kernel implements; this pins it
on the CPU, in fp64, before any kernel uses it: all chunk sizes, lengths that
are not multiples of the chunk, varlen packing, GQA, strongly negative gates
and beta up to 2.  Also the semantics the ABI promises: splitting a prompt at
any point and carrying the state equals the unsplit run; varlen equals
independent per-sequence runs.
"""
import numpy as np
import pytest

import oracle
from oracle import chunk_ref


def problem(rng, B, T, Hqk, Hv, dk, dv, g_scale=1.0, beta_max=2.0):
    q = rng.standard_normal((B, T, Hqk, dk))
    k = rng.standard_normal((B, T, Hqk, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, Hv, dv))
    g = g_scale * np.log(rng.uniform(0.5, 1.0, (B, T, Hv)))
    beta = rng.uniform(0, beta_max, (B, T, Hv))
    s0 = 0.1 * rng.standard_normal((B, Hv, dk, dv))
    return q, k, v, g, beta, s0


def rel(a, b):
    return np.max(np.abs(a - b)) / np.max(np.abs(b))


@pytest.mark.parametrize("C", [1, 2, 3, 8, 16, 64])
@pytest.mark.parametrize("T", [1, 7, 64, 65, 130])
def test_p6_chunk_form_equals_token_oracle(C, T):
    rng = np.random.default_rng(C * 1000 + T)
    prob = problem(rng, 1, T, 1, 2, 8, 4)
    o, s = oracle.run(*prob, scale=0.5)
    oc, sc = chunk_ref.run(*prob, scale=0.5, chunk=C)
    assert rel(oc, o) < 1e-10 and rel(sc, s) < 1e-10


def test_p6_strongly_negative_gates():
    rng = np.random.default_rng(11)
    q, k, v, g, beta, s0 = problem(rng, 1, 150, 1, 1, 8, 8)
    g = g * 200.0  # per-token log decay down to ~ -140: exp(-b_s) would overflow
    o, s = oracle.run(q, k, v, g, beta, s0)
    oc, sc = chunk_ref.run(q, k, v, g, beta, s0, chunk=64)
    assert np.all(np.isfinite(oc)) and np.all(np.isfinite(sc))
    np.testing.assert_allclose(oc, o, atol=1e-12 * np.max(np.abs(o)) + 1e-300)
    np.testing.assert_allclose(sc, s, atol=1e-12 * np.max(np.abs(s)) + 1e-300)


def test_p6_gqa_and_varlen():
    rng = np.random.default_rng(12)
    lens = [5, 64, 0, 129, 1]
    cu = np.cumsum([0] + lens)
    q, k, v, g, beta, _ = problem(rng, 1, int(cu[-1]), 2, 4, 16, 8)
    s0 = 0.1 * rng.standard_normal((len(lens), 4, 16, 8))
    o, s = oracle.run(q, k, v, g, beta, s0, cu_seqlens=cu)
    oc, sc = chunk_ref.run(q, k, v, g, beta, s0, cu_seqlens=cu, chunk=64)
    assert rel(oc, o) < 1e-10 and rel(sc, s) < 1e-10


def test_varlen_equals_independent_sequences():
    rng = np.random.default_rng(13)
    lens = [3, 17, 0, 9]
    cu = np.cumsum([0] + lens)
    q, k, v, g, beta, _ = problem(rng, 1, int(cu[-1]), 1, 2, 6, 5)
    s0 = rng.standard_normal((len(lens), 2, 6, 5))
    o, s = oracle.run(q, k, v, g, beta, s0, cu_seqlens=cu)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        on, sn = oracle.run(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], beta[:, a:b], s0[n:n + 1])
        np.testing.assert_array_equal(o[:, a:b], on)
        np.testing.assert_array_equal(s[n], sn[0])


@pytest.mark.parametrize("split", [1, 63, 64, 100])
def test_state_carry_equals_unsplit(split):
    rng = np.random.default_rng(14 + split)
    q, k, v, g, beta, s0 = problem(rng, 2, 160, 1, 1, 8, 8)
    o, s = oracle.run(q, k, v, g, beta, s0)
    sl = lambda a, lo, hi: a[:, lo:hi]
    o1, s1 = oracle.run(sl(q, 0, split), sl(k, 0, split), sl(v, 0, split), sl(g, 0, split),
                        sl(beta, 0, split), s0)
    o2, s2 = oracle.run(sl(q, split, 160), sl(k, split, 160), sl(v, split, 160),
                        sl(g, split, 160), sl(beta, split, 160), s1)
    np.testing.assert_array_equal(np.concatenate([o1, o2], axis=1), o)
    np.testing.assert_array_equal(s2, s)


def test_gqa_head_mapping_is_repeat_interleave():
    rng = np.random.default_rng(15)
    q, k, v, g, beta, s0 = problem(rng, 1, 20, 2, 6, 4, 3)
    o, s = oracle.run(q, k, v, g, beta, s0)
    qr = np.repeat(q, 3, axis=2)  # v-head h reads qk-head h // 3
    kr = np.repeat(k, 3, axis=2)
    o2, s2 = oracle.run(qr, kr, v, g, beta, s0)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(s, s2)


def test_decode_step_equals_one_token_prefill():
    rng = np.random.default_rng(16)
    q, k, v, g, beta, s0 = problem(rng, 3, 1, 2, 4, 8, 8)
    o, s = oracle.run(q, k, v, g, beta, s0)
    od, sd = oracle.step(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], s0)
    np.testing.assert_array_equal(od, o[:, 0])
    np.testing.assert_array_equal(sd, s)
