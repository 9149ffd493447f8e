"""Pins of the oracle's q/k L2 normalisation (qk_l2norm=True).

The normalisation is pinned by properties that a plausible mistake breaks:
- per-row positive rescaling of q and k changes nothing (fails if rows are not normalised,
  are divided by the squared norm, or are normalised over the wrong axis);
- on unit-norm rows the option is the identity;
- an all-zero key row is a token with no write (the beta = 0 invariant), and an all-zero
  query row reads zero.
"""
import numpy as np
import pytest

import oracle


def _inputs(B=2, T=37, Hqk=2, Hv=4, d=8, seed=0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, Hqk, d))
    k = rng.standard_normal((B, T, Hqk, d))
    v = rng.standard_normal((B, T, Hv, d))
    g = -rng.uniform(0.0, 0.5, (B, T, Hv))
    beta = rng.uniform(0.05, 1.9, (B, T, Hv))
    s0 = 0.1 * rng.standard_normal((B, Hv, d, d))
    return q, k, v, g, beta, s0


def test_row_rescaling_changes_nothing():
    q, k, v, g, beta, s0 = _inputs()
    rng = np.random.default_rng(1)
    cq = rng.uniform(0.01, 50.0, q.shape[:-1] + (1,))
    ck = rng.uniform(0.01, 50.0, k.shape[:-1] + (1,))
    o1, s1 = oracle.run(q, k, v, g, beta, s0, qk_l2norm=True)
    o2, s2 = oracle.run(q * cq, k * ck, v, g, beta, s0, qk_l2norm=True)
    assert np.abs(o1 - o2).max() <= 1e-12 * max(1.0, np.abs(o1).max())
    assert np.abs(s1 - s2).max() <= 1e-12 * max(1.0, np.abs(s1).max())
    # without the option the same rescaling does change the result
    o3, _ = oracle.run(q * cq, k * ck, v, g, beta, s0)
    assert np.abs(o3 - o1).max() > 1e-3


def test_identity_on_unit_rows():
    q, k, v, g, beta, s0 = _inputs(seed=2)
    q = q / np.linalg.norm(q, axis=-1, keepdims=True)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    o1, s1 = oracle.run(q, k, v, g, beta, s0, qk_l2norm=True)
    o2, s2 = oracle.run(q, k, v, g, beta, s0, qk_l2norm=False)
    assert np.abs(o1 - o2).max() <= 1e-13 and np.abs(s1 - s2).max() <= 1e-13


def test_zero_key_is_no_write_and_zero_query_reads_zero():
    q, k, v, g, beta, s0 = _inputs(B=1, T=9, Hqk=1, Hv=1, seed=3)
    t = 4
    kz = k.copy()
    kz[0, t] = 0.0
    bz = beta.copy()
    bz[0, t] = 0.0
    # k_t = 0 (normalised to 0) must equal beta_t = 0 with any key: only the decay applies
    o1, s1 = oracle.run(q, kz, v, g, beta, s0, qk_l2norm=True)
    o2, s2 = oracle.run(q, k, v, g, bz, s0, qk_l2norm=True)
    assert np.abs(s1 - s2).max() <= 1e-13
    # q_t = 0 reads zero at token t
    qz = q.copy()
    qz[0, t] = 0.0
    o3, _ = oracle.run(qz, k, v, g, beta, s0, qk_l2norm=True)
    assert np.abs(o3[0, t]).max() == 0.0


@pytest.mark.parametrize("form", [1, 2, 3])
def test_three_forms_agree_with_normalisation(form):
    q, k, v, g, beta, s0 = _inputs(seed=4)
    o1, s1 = oracle.run(q, k, v, g, beta, s0, form=2, qk_l2norm=True)
    o2, s2 = oracle.run(q, k, v, g, beta, s0, form=form, qk_l2norm=True)
    assert np.abs(o1 - o2).max() <= 1e-12 and np.abs(s1 - s2).max() <= 1e-12
