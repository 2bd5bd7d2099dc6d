"""Exact rational KDA: the definition as a product of explicit matrices.

TEST INFRASTRUCTURE (see the package docstring). For T <= 8 and tiny d.

This restates the definition (Kimi K3 technical FAQ, "What is KDA": delta rule
with a per-channel forget gate; standard gated-delta form) with nothing
rearranged: each token's transition is the explicit matrix
    M_t = (I - beta_t k_t k_t^T) Diag(alpha_t)
and the state after t tokens is the unrolled sum
    S_t = M_t ... M_1 S_0 + sum_{i<=t} (M_t ... M_{i+1}) beta_i k_i v_i^T,
    o_t = S_t^T q_t * scale.
Entries are fractions.Fraction, so the result is exact. alpha (not log alpha)
is the input here, which keeps it rational; the fp64 oracles take g = log alpha.
"""
from __future__ import annotations

from fractions import Fraction


def _eye(n):
    return [[Fraction(int(i == j)) for j in range(n)] for i in range(n)]


def _matmul(A, B):
    n, m, p = len(A), len(B), len(B[0])
    return [[sum((A[i][l] * B[l][j] for l in range(m)), Fraction(0)) for j in range(p)]
            for i in range(n)]


def _add(A, B):
    return [[a + b for a, b in zip(ra, rb)] for ra, rb in zip(A, B)]


def _outer(x, y, s=Fraction(1)):
    return [[s * a * b for b in y] for a in x]


def transition(k, alpha, beta):
    """M_t = (I - beta k k^T) Diag(alpha) as an explicit rational matrix."""
    n = len(k)
    I = _eye(n)
    P = [[I[i][j] - beta * k[i] * k[j] for j in range(n)] for i in range(n)]
    D = [[alpha[i] if i == j else Fraction(0) for j in range(n)] for i in range(n)]
    return _matmul(P, D)


def kda_exact(q, k, v, alpha, beta, s0, scale):
    """Exact outputs and states of one head.

    q, k, alpha: T lists of dk Fractions; v: T lists of dv Fractions; beta: T
    Fractions; s0: dk x dv Fractions; scale: a Fraction.
    Returns (o: T lists of dv Fractions, states: T dk x dv matrices S_1..S_T).
    """
    T = len(k)
    M = [transition(k[t], alpha[t], beta[t]) for t in range(T)]
    outs, states = [], []
    for t in range(T):
        # P(t, i) = M_t ... M_{i+1}; P(t, t) = I
        P = [None] * (t + 2)
        P[t + 1] = _eye(len(k[0]))
        for i in range(t, -1, -1):
            P[i] = _matmul(P[i + 1], M[i])
        # P[i] now holds M_t ... M_i (0-based tokens); the term for token i uses
        # the product of the later transitions, P[i + 1].
        S = _matmul(P[0], s0)
        for i in range(t + 1):
            S = _add(S, _matmul(P[i + 1], _outer(k[i], v[i], beta[i])))
        o = [scale * sum((S[a][j] * q[t][a] for a in range(len(q[t]))), Fraction(0))
             for j in range(len(v[t]))]
        outs.append(o)
        states.append(S)
    return outs, states
