"""numpy fp64 oracle of the q/k front-end of a KDA layer.

TEST INFRASTRUCTURE (see the package docstring).

Kimi K3 technical FAQ, "What is KDA": queries and keys pass through a short
convolution, Swish and L2 normalisation before the recurrence. The page gives
no further detail; the readings taken here (stated in the design notes):
  - the short convolution is causal and depthwise over time: each channel c of
    head h has K taps w[h, c, 0..K-1], and
        y_t = sum_{j=0}^{K-1} w[h, c, j] * x_{t-(K-1)+j}
    so tap K-1 multiplies the current token; no bias;
  - inputs before a sequence's first token come from its conv state, the last
    K-1 inputs of the previous segment (zeros for a fresh sequence), and the
    state after a segment is its last K-1 inputs (prefix caching keeps it with
    the recurrent state at the same block boundaries);
  - Swish(y) = y * sigmoid(y);
  - L2 normalisation over the d_k channels of each (token, head):
    z / max(||z||_2, eps), eps = 1e-6.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def short_conv(x: np.ndarray, w: np.ndarray, state: np.ndarray | None = None):
    """Causal depthwise convolution of one sequence.

    x [T, H, D]; w [H, D, K]; state [H, D, K-1] or None (zeros): the inputs at
    times -(K-1) .. -1. Returns (y [T, H, D], new_state [H, D, K-1]) where
    new_state holds the inputs at times T-(K-1) .. T-1 (older ones from `state`
    when T < K-1)."""
    T, H, D = x.shape
    K = w.shape[-1]
    hist = np.zeros((H, D, K - 1)) if state is None else np.asarray(state, dtype=np.float64)
    # xs[i] is the input at time i - (K-1)
    xs = np.concatenate([np.moveaxis(hist, -1, 0), np.asarray(x, dtype=np.float64)], axis=0)
    y = np.zeros((T, H, D))
    for t in range(T):
        for j in range(K):
            y[t] += w[:, :, j] * xs[t + j]
    new_state = np.moveaxis(xs[T:T + K - 1], 0, -1).copy()
    return y, new_state


def swish(y: np.ndarray) -> np.ndarray:
    """y * sigmoid(y), written as y / (1 + exp(-y)) with the exponent clipped so
    that very negative y gives 0 instead of an overflow warning."""
    return y / (1.0 + np.exp(np.minimum(-y, 700.0)))


def l2_normalise(z: np.ndarray, eps: float = EPS) -> np.ndarray:
    """z / max(||z||_2, eps) over the last axis."""
    n = np.sqrt(np.sum(z * z, axis=-1, keepdims=True))
    return z / np.maximum(n, eps)


def qk_frontend(x: np.ndarray, w: np.ndarray, state: np.ndarray | None = None):
    """L2(Swish(short_conv(x))) for one sequence: returns (features [T, H, D],
    new conv state [H, D, K-1])."""
    y, new_state = short_conv(x, w, state)
    return l2_normalise(swish(y)), new_state


def qk_frontend_packed(x, cu_seqlens, w, states=None, start_pos=None, snap_interval=0):
    """Packed ragged batch: sequence s is rows cu[s]..cu[s+1]-1 of x [T, H, D].
    states [n_seq, H, D, K-1] (None: zeros). Returns (features [T, H, D],
    final conv states [n_seq, H, D, K-1], conv-state snapshots [n_snap, H, D, K-1])
    with snapshots after each absolute position p with start_pos < p <=
    start_pos + len and p % snap_interval == 0, sequence by sequence, ascending
    (the rule of the recurrent-state snapshots)."""
    cu = np.asarray(cu_seqlens)
    n_seq = len(cu) - 1
    H, D, K = w.shape
    out = np.zeros(x.shape)
    finals = np.zeros((n_seq, H, D, K - 1))
    snaps = []
    for s in range(n_seq):
        a, b = int(cu[s]), int(cu[s + 1])
        p0 = 0 if start_pos is None else int(start_pos[s])
        st = None if states is None else states[s]
        feats, fin = qk_frontend(x[a:b], w, st)
        out[a:b] = feats
        finals[s] = fin
        if snap_interval > 0:
            for p in range((p0 // snap_interval + 1) * snap_interval, p0 + (b - a) + 1, snap_interval):
                _, st_p = short_conv(x[a:a + p - p0], w, st)
                snaps.append(st_p)
    snaps = np.stack(snaps) if snaps else np.zeros((0, H, D, K - 1))
    return out, finals, snaps
