"""Pins of the q/k front-end oracle (oracle/frontend.py): short causal depthwise
convolution, Swish and L2 normalisation (Kimi K3 technical FAQ, "What is KDA").
Each pin checks the oracle against something other than itself: a library routine
(numpy.correlate, scipy.special.expit, numpy.linalg.norm), a closed form (delta
taps), or brute-force slicing of the inputs for the carried conv state.
"""
from __future__ import annotations

import numpy as np
import pytest
from scipy.special import expit

from oracle import frontend as F
from oracle.recurrence import snapshot_count


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("K", [2, 3, 4])
def test_conv_equals_numpy_correlate_over_state_and_inputs(K):
    rng = _rng(K)
    T, H, D = 13, 2, 5
    x = rng.standard_normal((T, H, D))
    w = rng.standard_normal((H, D, K))
    st = rng.standard_normal((H, D, K - 1))
    y, new = F.short_conv(x, w, st)
    for h in range(H):
        for c in range(D):
            xs = np.concatenate([st[h, c], x[:, h, c]])     # times -(K-1) .. T-1
            ref = np.correlate(xs, w[h, c], mode="valid")   # sum_j xs[t + j] w[j]
            assert np.allclose(y[:, h, c], ref, rtol=0, atol=1e-13)
            assert np.array_equal(new[h, c], xs[-(K - 1):])


def test_conv_delta_taps():
    """Tap K-1 alone is the identity; tap 0 alone delays by K-1 tokens, reading the
    carried state for the first K-1 outputs."""
    rng = _rng(7)
    T, H, D, K = 9, 3, 4, 4
    x = rng.standard_normal((T, H, D))
    st = rng.standard_normal((H, D, K - 1))
    w = np.zeros((H, D, K))
    w[..., K - 1] = 1.0
    y, _ = F.short_conv(x, w, st)
    assert np.array_equal(y, x)
    w = np.zeros((H, D, K))
    w[..., 0] = 1.0
    y, _ = F.short_conv(x, w, st)
    assert np.array_equal(y[K - 1:], x[:T - (K - 1)])
    for t in range(K - 1):
        assert np.array_equal(y[t], st[..., t])


def test_conv_without_state_reads_zeros_and_short_segments_keep_old_state():
    rng = _rng(8)
    H, D, K = 2, 3, 4
    w = rng.standard_normal((H, D, K))
    x = rng.standard_normal((2, H, D))                     # shorter than K - 1
    st = rng.standard_normal((H, D, K - 1))
    _, new = F.short_conv(x, w, st)
    assert np.array_equal(new[..., 0], st[..., 2])         # oldest kept input
    assert np.array_equal(new[..., 1:], np.moveaxis(x, 0, -1))
    y0, _ = F.short_conv(x, w, None)
    y1, _ = F.short_conv(x, w, np.zeros((H, D, K - 1)))
    assert np.array_equal(y0, y1)


def test_segments_equal_one_pass():
    """Carrying the conv state across a split gives the one-pass result."""
    rng = _rng(9)
    T, H, D, K = 20, 2, 6, 4
    x = rng.standard_normal((T, H, D))
    w = rng.standard_normal((H, D, K))
    full, fin = F.short_conv(x, w)
    for cut in (1, 2, 3, 7, 19):
        a, st = F.short_conv(x[:cut], w)
        b, fin2 = F.short_conv(x[cut:], w, st)
        assert np.allclose(np.concatenate([a, b]), full, rtol=0, atol=1e-13)
        assert np.array_equal(fin2, fin)


def test_swish_against_expit_and_limits():
    y = np.linspace(-30, 30, 601)
    assert np.allclose(F.swish(y), y * expit(y), rtol=1e-13, atol=1e-300)
    assert F.swish(np.array([0.0]))[0] == 0.0
    assert abs(F.swish(np.array([40.0]))[0] - 40.0) < 1e-15
    assert 0.0 >= F.swish(np.array([-800.0]))[0] > -1e-300


def test_l2_normalise_unit_norm_scale_invariance_and_zero_rows():
    rng = _rng(10)
    z = rng.standard_normal((5, 3, 16))
    n = F.l2_normalise(z)
    assert np.allclose(np.linalg.norm(n, axis=-1), 1.0, rtol=0, atol=1e-14)
    assert np.allclose(n, z / np.linalg.norm(z, axis=-1, keepdims=True), rtol=0, atol=1e-15)
    assert np.allclose(F.l2_normalise(3.5 * z), n, rtol=0, atol=1e-15)
    zero = np.zeros((2, 16))
    assert np.array_equal(F.l2_normalise(zero), zero)
    tiny = np.full((1, 4), 1e-9)                           # norm below eps: divided by eps
    assert np.allclose(F.l2_normalise(tiny), tiny / F.EPS)


def test_frontend_composition_order():
    """conv, then Swish, then L2: with the identity tap the front-end is
    L2(Swish(x)); the features have unit norm per (token, head)."""
    rng = _rng(11)
    T, H, D, K = 6, 2, 8, 4
    x = rng.standard_normal((T, H, D))
    w = np.zeros((H, D, K))
    w[..., K - 1] = 1.0
    f, _ = F.qk_frontend(x, w)
    s = x * expit(x)
    assert np.allclose(f, s / np.linalg.norm(s, axis=-1, keepdims=True), rtol=0, atol=1e-14)


def test_packed_batch_states_and_snapshots_by_brute_force():
    """Per-sequence results equal single-sequence calls; each conv-state snapshot is
    the last K-1 inputs up to its position (older ones from the initial state)."""
    rng = _rng(12)
    H, D, K, interval = 2, 4, 4, 4
    lens = [0, 3, 9, 12]
    start = [4, 0, 8, 2]
    cu = np.concatenate([[0], np.cumsum(lens)])
    x = rng.standard_normal((int(cu[-1]), H, D))
    w = rng.standard_normal((H, D, K))
    st = rng.standard_normal((len(lens), H, D, K - 1))
    out, fins, snaps = F.qk_frontend_packed(x, cu, w, st, start, interval)
    assert snaps.shape[0] == sum(snapshot_count(p, n, interval) for p, n in zip(start, lens))
    row = 0
    for s, (n, p0) in enumerate(zip(lens, start)):
        a, b = int(cu[s]), int(cu[s + 1])
        f1, fin1 = F.qk_frontend(x[a:b], w, st[s])
        assert np.array_equal(out[a:b], f1)
        assert np.array_equal(fins[s], fin1)
        hist = np.concatenate([np.moveaxis(st[s], -1, 0), x[a:b]])   # times -(K-1) .. n-1
        for p in range(p0 + 1, p0 + n + 1):
            if p % interval:
                continue
            m = p - p0                                     # tokens of this call consumed
            assert np.array_equal(snaps[row], np.moveaxis(hist[m:m + K - 1], 0, -1))
            row += 1
    assert row == snaps.shape[0]
