"""Pins of the segment state maps (oracle/segments.py): the affine map of a run of
tokens, its composition, and the two-pass split of one sequence (the algebra of
context-parallel prefill). Checked against the token recurrence (itself pinned in
test_oracle_pins.py) and against closed forms of the definition (Kimi K3 technical
FAQ, "What is KDA"; standard gated-delta form).
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle import segments as SG
from oracle.recurrence import kda_recurrence


def _inputs(seed, T, dk=8, dv=6):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, 1, dk))
    k = rng.standard_normal((T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, 1, dv))
    g = -0.2 * np.log1p(np.exp(rng.standard_normal((T, 1, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, 1))))
    return q, k, v, g, beta


def test_map_reproduces_the_recurrence_from_any_state():
    q, k, v, g, beta = _inputs(1, 23)
    M, N = SG.segment_map(k[:, 0], v[:, 0], g[:, 0], beta[:, 0])
    rng = np.random.default_rng(2)
    for _ in range(3):
        S0 = rng.standard_normal((8, 6))
        _, S, _ = kda_recurrence(q, k, v, g, beta, S0[None])
        assert np.allclose(SG.apply((M, N), S0), S[0], rtol=0, atol=1e-12)
    _, S, _ = kda_recurrence(q, k, v, g, beta)
    assert np.allclose(N, S[0], rtol=0, atol=1e-12)      # N is the final state from zero


def test_beta_zero_gives_the_decay_alone():
    q, k, v, g, beta = _inputs(3, 11)
    M, N = SG.segment_map(k[:, 0], v[:, 0], g[:, 0], np.zeros(11))
    assert np.allclose(M, np.diag(np.exp(g[:, 0].sum(axis=0))), rtol=1e-13, atol=0)
    assert np.array_equal(N, np.zeros_like(N))


def test_orthonormal_overwrites_give_a_projector():
    """alpha = 1, beta = 1 and orthonormal keys: M = I - sum k k^T, N = sum k v^T."""
    rng = np.random.default_rng(4)
    dk, dv, T = 8, 5, 5
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :T].T
    v = rng.standard_normal((T, dv))
    M, N = SG.segment_map(k, v, np.zeros((T, dk)), np.ones(T))
    assert np.allclose(M, np.eye(dk) - k.T @ k, rtol=0, atol=1e-13)
    assert np.allclose(N, k.T @ v, rtol=0, atol=1e-13)


@pytest.mark.parametrize("cuts", [[7], [1, 2, 30], [5, 11, 19, 24]])
def test_composition_equals_the_map_of_the_concatenation(cuts):
    q, k, v, g, beta = _inputs(5, 31)
    args = (k[:, 0], v[:, 0], g[:, 0], beta[:, 0])
    whole = SG.segment_map(*args)
    bounds = [0] + cuts + [31]
    maps = [SG.segment_map(*(a[lo:hi] for a in args)) for lo, hi in zip(bounds[:-1], bounds[1:])]
    acc = maps[0]
    for m in maps[1:]:
        acc = SG.compose(m, acc)
    assert np.allclose(acc[0], whole[0], rtol=0, atol=1e-12)
    assert np.allclose(acc[1], whole[1], rtol=0, atol=1e-12)
    # associativity of the composition
    if len(maps) >= 3:
        left = SG.compose(maps[2], SG.compose(maps[1], maps[0]))
        right = SG.compose(SG.compose(maps[2], maps[1]), maps[0])
        assert np.allclose(left[0], right[0], rtol=0, atol=1e-13)
        assert np.allclose(left[1], right[1], rtol=0, atol=1e-13)


def test_two_pass_split_reproduces_outputs_and_final_state():
    """Pass 1: each segment's map, from zero. Scan: the state entering each segment.
    Pass 2: each segment's recurrence from its entering state. Together they equal
    the one-pass recurrence of the whole sequence."""
    q, k, v, g, beta = _inputs(6, 40)
    rng = np.random.default_rng(7)
    S0 = rng.standard_normal((8, 6))
    o_ref, S_ref, _ = kda_recurrence(q, k, v, g, beta, S0[None])
    bounds = [0, 9, 10, 27, 40]
    maps = [SG.segment_map(k[lo:hi, 0], v[lo:hi, 0], g[lo:hi, 0], beta[lo:hi, 0])
            for lo, hi in zip(bounds[:-1], bounds[1:])]
    entering, S_end = SG.entering_states(maps, S0)
    assert np.allclose(S_end, S_ref[0], rtol=0, atol=1e-12)
    for (lo, hi), Sin in zip(zip(bounds[:-1], bounds[1:]), entering):
        o, _, _ = kda_recurrence(q[lo:hi], k[lo:hi], v[lo:hi], g[lo:hi], beta[lo:hi], Sin[None])
        assert np.allclose(o, o_ref[lo:hi], rtol=0, atol=1e-12)
