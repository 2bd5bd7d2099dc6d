"""numpy fp64 oracle of segment state maps (the algebra of splitting one long
sequence across workers).

TEST INFRASTRUCTURE (see the package docstring). Small cases only.

Each step of the recurrence (Kimi K3 technical FAQ, "What is KDA"; standard
gated-delta form) is affine in the state:
    S_t = A_t S_{t-1} + B_t,   A_t = (I - beta_t k_t k_t^T) Diag(alpha_t)  (d_k x d_k),
                               B_t = beta_t k_t v_t^T                     (d_k x d_v).
So a segment of tokens t0 .. t1-1 maps the state entering it to the state
leaving it by S_{t1} = M S_{t0} + N, with
    M = A_{t1-1} ... A_{t0},   N = sum_t (A_{t1-1} ... A_{t+1}) B_t,
and segment maps compose as (M2, N2) o (M1, N1) = (M2 M1, M2 N1 + N2). N alone is
the segment's final state from a zero state. A worker that holds one segment can
therefore compute (M, N) without knowing the state before it; an exclusive scan
of the maps gives every segment's entering state, and each segment's outputs
follow from a second pass that starts from it.
"""
from __future__ import annotations

import numpy as np


def step_map(k, v, g, beta):
    """(A_t, B_t) of one token of one head: k, g [d_k]; v [d_v]; beta scalar."""
    k = np.asarray(k, dtype=np.float64)
    dk = k.shape[0]
    A = (np.eye(dk) - beta * np.outer(k, k)) @ np.diag(np.exp(np.asarray(g, dtype=np.float64)))
    B = beta * np.outer(k, np.asarray(v, dtype=np.float64))
    return A, B


def segment_map(k, v, g, beta):
    """(M, N) of a segment of one head: k, g [T, d_k]; v [T, d_v]; beta [T]."""
    T, dk = k.shape
    M = np.eye(dk)
    N = np.zeros((dk, v.shape[1]))
    for t in range(T):
        A, B = step_map(k[t], v[t], g[t], beta[t])
        M = A @ M
        N = A @ N + B
    return M, N


def compose(second, first):
    """The map of `first` followed by `second`."""
    M2, N2 = second
    M1, N1 = first
    return M2 @ M1, M2 @ N1 + N2


def apply(seg, S):
    M, N = seg
    return M @ S + N


def entering_states(maps, S0):
    """Exclusive scan: the state entering each segment, given the state S0 before the
    first one."""
    out = []
    S = np.asarray(S0, dtype=np.float64)
    for seg in maps:
        out.append(S)
        S = apply(seg, S)
    return out, S
