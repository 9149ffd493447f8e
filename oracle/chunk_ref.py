"""numpy fp64 chunk (UT/WY) form of the gated delta rule.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

This restates the chunkwise-parallel form named by "Parallelizing Linear
Transformers with the Delta Rule over Sequence Length" (title cited on the
"DeltaNet Attention" and "DeltaNet" pages) with the per-token decay of the
"linear_attention" page folded in.  The pages give only the token recurrence;
the chunk algebra below is derived from it and is pinned against the token
oracle (``tests/test_oracle_chunk.py``) for many chunk sizes and ragged tails.

Stored state H = S^T (d_k x d_v).  Token recurrence in stored form:
    H_t = alpha_t (I - beta_t k_t k_t^T) H_{t-1} + beta_t k_t v_t^T,   o_t = H_t^T q_t.
For one chunk of L tokens starting from H0 (rows r, s = 0..L-1):
    b_r = sum_{i<=r} g_i,  gamma_r = exp(b_r),  Gamma_rs = exp(b_r - b_s) (s <= r, else 0)
    Lmat = strict_lower(diag(beta) (Gamma * K K^T)),   T = (I + Lmat)^-1
    W = T diag(beta gamma) K,    U = T diag(beta) V,    Delta = U - W H0
    O = diag(gamma) Q H0 + (Gamma * Q K^T * incl_lower) Delta
    H_L = gamma_{L-1} H0 + Ktil^T Delta,   Ktil_s = exp(b_{L-1} - b_s) k_s
"""
from __future__ import annotations

import numpy as np


def chunk_step(Q, K, V, g, beta, H0):
    """One chunk.  Q, K: [L, dk]; V: [L, dv]; g, beta: [L]; H0: [dk, dv].

    Returns (O [L, dv], H_L [dk, dv]).  All float64.
    """
    L = K.shape[0]
    b = np.cumsum(g)
    gamma = np.exp(b)
    diff = b[:, None] - b[None, :]
    incl = np.tril(np.ones((L, L), dtype=bool))
    Gam = np.where(incl, np.exp(np.where(incl, diff, 0.0)), 0.0)
    A = K @ K.T
    Lmat = np.tril(beta[:, None] * Gam * A, k=-1)
    T = np.linalg.inv(np.eye(L) + Lmat)
    W = T @ ((beta * gamma)[:, None] * K)
    U = T @ (beta[:, None] * V)
    Delta = U - W @ H0
    P = Gam * (Q @ K.T)  # Gam is already zero above the diagonal
    O = gamma[:, None] * (Q @ H0) + P @ Delta
    Ktil = np.exp(b[-1] - b)[:, None] * K
    H1 = gamma[-1] * H0 + Ktil.T @ Delta
    return O, H1


def chunk_step_channel(Q, K, V, g, beta, H0):
    """One chunk with per-key-channel gates g [L, dk] (the "linear_attention" page's
    ChannelGates).  Same returns as ``chunk_step``.

    With b_r = sum_{i<=r} g_i now a vector, the decay between tokens s <= r is
    diag(exp(b_r - b_s)) and no longer factors out of the key products:
        A_rs = sum_c k_r[c] k_s[c] exp(b_r[c] - b_s[c]),   Lmat = strict_lower(diag(beta) A)
        W = T diag(beta) (K o e^b),   U = T diag(beta) V,   Delta = U - W H0
        P_rs = sum_c q_r[c] k_s[c] exp(b_r[c] - b_s[c]) (s <= r)
        O = (Q o e^b) H0 + P Delta,   H_L = diag(e^{b_{L-1}}) H0 + (K o e^{b_{L-1} - b})^T Delta
    (o: elementwise, rows broadcast).  The scalar form is the case of equal columns.
    """
    L = K.shape[0]
    b = np.cumsum(g, axis=0)                              # [L, dk]
    incl = np.tril(np.ones((L, L), dtype=bool))
    diff = b[:, None, :] - b[None, :, :]                  # [L, L, dk], r - s
    E = np.where(incl[:, :, None], np.exp(np.where(incl[:, :, None], diff, 0.0)), 0.0)
    A = np.einsum("rc,sc,rsc->rs", K, K, E)
    Lmat = np.tril(beta[:, None] * A, k=-1)
    T = np.linalg.inv(np.eye(L) + Lmat)
    W = T @ (beta[:, None] * (K * np.exp(b)))
    U = T @ (beta[:, None] * V)
    Delta = U - W @ H0
    P = np.einsum("rc,sc,rsc->rs", Q, K, E)
    O = (Q * np.exp(b)) @ H0 + P @ Delta
    H1 = np.exp(b[-1])[:, None] * H0 + (K * np.exp(b[-1] - b)).T @ Delta
    return O, H1


def run(q, k, v, g, beta, state_in=None, cu_seqlens=None, scale=1.0, chunk=64,
        chunk_states=False):
    """Chunk form over a whole (possibly varlen-packed) batch.

    Same layouts and return values as ``oracle.run``.  The last chunk of a
    sequence may be shorter than ``chunk``.  With ``chunk_states`` a third array
    holds H_L of every chunk, sequence after sequence (the rows ``oracle.run`` with
    ``chunk_len=chunk`` returns).
    """
    q, k, v, beta = (np.asarray(a, dtype=np.float64) for a in (q, k, v, beta))
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    g = np.zeros((B, T, Hv)) if g is None else np.asarray(g, dtype=np.float64)
    step = chunk_step_channel if g.ndim == 4 else chunk_step
    if cu_seqlens is not None:
        cu = [int(x) for x in np.asarray(cu_seqlens)]
        seqs = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    else:
        seqs = [(b_, 0, T) for b_ in range(B)]
    N = len(seqs)
    group = Hv // Hqk
    o = np.zeros((B, T, Hv, dv))
    st = np.zeros((N, Hv, dk, dv))
    rows = [(n, c0) for n, (bb, t0, t1) in enumerate(seqs) for c0 in range(t0, t1, chunk)]
    cs = np.zeros((len(rows), Hv, dk, dv))
    for n, (bb, t0, t1) in enumerate(seqs):
        for h in range(Hv):
            hq = h // group
            H = np.zeros((dk, dv)) if state_in is None else np.array(state_in[n, h], dtype=np.float64)
            for c0 in range(t0, t1, chunk):
                c1 = min(c0 + chunk, t1)
                O, H = step(scale * q[bb, c0:c1, hq], k[bb, c0:c1, hq], v[bb, c0:c1, h],
                            g[bb, c0:c1, h], beta[bb, c0:c1, h], H)
                o[bb, c0:c1, h] = O
                cs[rows.index((n, c0)), h] = H
            st[n, h] = H
    return (o, st, cs) if chunk_states else (o, st)
