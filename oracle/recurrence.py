"""numpy fp64 KDA oracle: token recurrence, snapshot rule and chunked form.

TEST INFRASTRUCTURE (see the package docstring). Small cases only.

Token recurrence (Kimi K3 technical FAQ, "What is KDA": delta rule with a
per-channel forget gate; standard gated-delta form):
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
    o_t = scale * S_t^T q_t,   alpha_t = exp(g_t) (per key channel)

Chunked form (the same FAQ: "parallel within a chunk, recurrent across
chunks"). The pages give no algebra; this is derived from the recurrence. Put
D_t = Diag(alpha_t), b_r = sum_{i<=r} g_i inside a chunk (inclusive), Gamma_r =
exp(b_r). Writing S_t = D_t S_{t-1} + k_t w_t^T with
w_t = beta_t (v_t - S_{t-1}^T D_t k_t) and unrolling from the chunk start S_0:
    S_r = Diag(Gamma_r) S_0 + sum_{i<=r} Diag(Gamma_r / Gamma_i) k_i w_i^T
    (I + Diag(beta) A_kk) W = Diag(beta) (V - (K . Gamma) S_0)
    A_kk[r, i] = sum_c k_rc k_ic exp(b_rc - b_ic),  i < r
    O = scale * [ (Q . Gamma) S_0 + A_qk W ],
    A_qk[r, i] = sum_c q_rc k_ic exp(b_rc - b_ic),  i <= r
    S_C = Diag(Gamma_C) S_0 + (K . exp(b_C - b))^T W
Here every exponent is a difference b_r - b_i with i <= r, so it is <= 0.
"""
from __future__ import annotations

import numpy as np


def snapshot_count(start_pos: int, length: int, interval: int) -> int:
    """Number of absolute positions p with start_pos < p <= start_pos+length and
    p % interval == 0 (state after p tokens; vLLM day-0 blog, state snapshots at
    block boundaries)."""
    if interval <= 0:
        return 0
    return (start_pos + length) // interval - start_pos // interval


def snapshot_positions(start_pos: int, length: int, interval: int) -> list[int]:
    """The absolute positions of those snapshots, ascending."""
    if interval <= 0:
        return []
    first = (start_pos // interval + 1) * interval
    return list(range(first, start_pos + length + 1, interval))


def kda_recurrence(q, k, v, g, beta, s0=None, scale=None, start_pos=0, snap_interval=0):
    """Token-by-token fp64 recurrence for one sequence, all heads.

    q, k, g: [T, H, dk]; v: [T, H, dv]; beta: [T, H]; s0: [H, dk, dv] or None.
    Returns (o [T, H, dv], s_final [H, dk, dv], snaps [n, H, dk, dv]) in fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    T, H, dk = k.shape
    dv = v.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    S = np.zeros((H, dk, dv)) if s0 is None else np.array(s0, dtype=np.float64)
    o = np.zeros((T, H, dv))
    snaps = []
    for t in range(T):
        S = np.exp(g[t])[:, :, None] * S                        # Diag(alpha_t) S
        x = np.einsum("hij,hi->hj", S, k[t])                    # S^T k_t
        S = S + beta[t][:, None, None] * k[t][:, :, None] * (v[t] - x)[:, None, :]
        o[t] = scale * np.einsum("hij,hi->hj", S, q[t])         # S_t^T q_t
        p = start_pos + t + 1
        if snap_interval > 0 and p % snap_interval == 0:
            snaps.append(S.copy())
    snaps = np.stack(snaps) if snaps else np.zeros((0, H, dk, dv))
    return o, S, snaps


def kda_chunked(q, k, v, g, beta, s0=None, scale=None, chunk=64, start_pos=0,
                snap_interval=0):
    """The chunked (WY/UT) form of the same map, fp64, one sequence, all heads.

    Chunks start at the sequence's first token of this call; the last chunk may
    be short. Snapshots are taken at chunk ends whose absolute position is a
    multiple of snap_interval (requires snap_interval % chunk == 0 and
    start_pos % chunk == 0 when snapshots are requested).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    T, H, dk = k.shape
    dv = v.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    if snap_interval > 0:
        assert snap_interval % chunk == 0 and start_pos % chunk == 0
    S = np.zeros((H, dk, dv)) if s0 is None else np.array(s0, dtype=np.float64)
    o = np.zeros((T, H, dv))
    snaps = []
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        n = c1 - c0
        Q = q[c0:c1].transpose(1, 0, 2)        # [H, n, dk]
        K = k[c0:c1].transpose(1, 0, 2)
        V = v[c0:c1].transpose(1, 0, 2)        # [H, n, dv]
        B = beta[c0:c1].T                      # [H, n]
        b = np.cumsum(g[c0:c1].transpose(1, 0, 2), axis=1)   # [H, n, dk] inclusive
        Gam = np.exp(b)
        # pairwise decays exp(b_rc - b_ic), used only where i <= r
        diff = b[:, :, None, :] - b[:, None, :, :]             # [H, r, i, c]
        tril_incl = np.tril(np.ones((n, n), dtype=bool))
        tril_strict = np.tril(np.ones((n, n), dtype=bool), -1)
        E = np.where(tril_incl[None, :, :, None], np.exp(np.minimum(diff, 0.0)), 0.0)
        A_kk = np.einsum("hrc,hic,hric->hri", K, K, E) * tril_strict
        A_qk = np.einsum("hrc,hic,hric->hri", Q, K, E) * tril_incl
        L = np.eye(n)[None] + B[:, :, None] * A_kk             # I + Diag(beta) A_kk
        rhs = B[:, :, None] * (V - np.einsum("hrc,hcj->hrj", K * Gam, S))
        W = np.linalg.solve(L, rhs)                            # [H, n, dv]
        o[c0:c1] = (scale * (np.einsum("hrc,hcj->hrj", Q * Gam, S)
                             + np.einsum("hri,hij->hrj", A_qk, W))).transpose(1, 0, 2)
        bC = b[:, -1, :]                                        # [H, dk]
        S = np.exp(bC)[:, :, None] * S + np.einsum("hic,hij->hcj", K * np.exp(bC[:, None, :] - b), W)
        p = start_pos + c1
        if snap_interval > 0 and p % snap_interval == 0:
            snaps.append(S.copy())
    snaps = np.stack(snaps) if snaps else np.zeros((0, H, dk, dv))
    return o, S, snaps


def normwise_rel_err(x, ref, axes=None):
    """max|x - ref| / max|ref| over each block; blocks are the leading axes not
    in ``axes`` (default: the whole array is one block). Returns the max over
    blocks (the tolerance metric of the KDA parity tests)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if axes is None:
        den = np.max(np.abs(ref))
        return float(np.max(np.abs(x - ref)) / den) if den > 0 else float(np.max(np.abs(x)))
    num = np.max(np.abs(x - ref), axis=axes)
    den = np.max(np.abs(ref), axis=axes)
    den = np.where(den > 0, den, 1.0)
    return float(np.max(num / den))
