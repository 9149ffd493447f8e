"""Exact rational brute force for tiny inputs.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The delta-rule update of the "DeltaNet Attention" page,
S_t = S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T, with the per-token decay
alpha_t of the "linear_attention" page, is affine in S.  Writing
A_t = alpha_t (I - beta_t k_t k_t^T), its solution is the closed product

    S_t = S_0 A_1 ... A_t + sum_{s<=t} beta_s v_s k_s^T A_{s+1} ... A_t,
    o_t = S_t q_t,

evaluated here with ``fractions.Fraction`` (no rounding at all) by forming the
products explicitly, never by stepping the recurrence.  alpha_t is supplied
directly as a rational number (exp(g) is not rational).  With per-key-channel
gates (the "linear_attention" page's ChannelGates) alpha_t is a vector and
A_t = diag(alpha_t) (I - beta_t k_t k_t^T).
"""
from __future__ import annotations

from fractions import Fraction


def _matmul(X, Y):
    n, m, p = len(X), len(Y), len(Y[0])
    return [[sum((X[i][a] * Y[a][j] for a in range(m)), Fraction(0)) for j in range(p)]
            for i in range(n)]


def _eye(n):
    return [[Fraction(int(i == j)) for j in range(n)] for i in range(n)]


def solve(q, k, v, alpha, beta, S0):
    """q, k: T x dk; v: T x dv; alpha, beta: T; S0: dv x dk (all Fractions).

    alpha[t] may be a list of dk Fractions (one decay per key channel).

    Returns (o: T x dv, S_T: dv x dk), exact.
    """
    T = len(k)
    dk = len(k[0])
    dv = len(v[0])
    A = []
    for t in range(T):
        al = alpha[t] if isinstance(alpha[t], (list, tuple)) else [alpha[t]] * dk
        At = [[al[a] * ((1 if a == b else 0) - beta[t] * k[t][a] * k[t][b]) for b in range(dk)]
              for a in range(dk)]
        A.append(At)

    def prod(a, b):  # A_a ... A_b (1-based, inclusive); identity when a > b
        P = _eye(dk)
        for t in range(a, b + 1):
            P = _matmul(P, A[t - 1])
        return P

    o = []
    S = None
    for t in range(1, T + 1):
        S = _matmul(S0, prod(1, t))
        for s in range(1, t + 1):
            outer = [[beta[s - 1] * v[s - 1][j] * k[s - 1][i] for i in range(dk)] for j in range(dv)]
            term = _matmul(outer, prod(s + 1, t))
            S = [[S[j][i] + term[j][i] for i in range(dk)] for j in range(dv)]
        o.append([sum((S[j][i] * q[t - 1][i] for i in range(dk)), Fraction(0)) for j in range(dv)])
    if S is None:
        S = [row[:] for row in S0]
    return o, S
