"""Pins for the CPU oracle: each check compares the oracle with something other
than itself -- the exact rational product form, closed forms, exact special
cases of the definition and invariants it implies.

Definition (Kimi K3 technical FAQ, "What is KDA": delta rule with a
per-channel forget gate, d_k x d_v state per head; standard gated-delta form):
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
    o_t = S_t^T q_t * scale
Snapshots (vLLM day-0 blog, "Kimi Delta Attention": state snapshots at block
boundaries): the state after absolute position p, p % interval == 0.

Every pin runs on each oracle implementation (numpy token loop, C token loop,
numpy chunked form at several chunk sizes). The last test plants mistakes in a
copy of the oracle (on the CPU) and checks that some pin catches each one.
"""
from __future__ import annotations

import json
from fractions import Fraction
from pathlib import Path

import numpy as np
import pytest

import synth
from oracle import native
from oracle.recurrence import (kda_chunked, kda_recurrence, normwise_rel_err,
                               snapshot_count, snapshot_positions)

GOLDEN = Path(__file__).resolve().parent / "golden" / "exact_product_T8_d4.json"


# --------------------------------------------------------------------------
# implementations under test: run(q,k,v,g,beta,s0,scale,start_pos,snap) ->
# (o, S_final, snaps or None when the implementation cannot snapshot there)
# --------------------------------------------------------------------------
def run_numpy(q, k, v, g, beta, s0=None, scale=None, start_pos=0, snap=0):
    return kda_recurrence(q, k, v, g, beta, s0, scale, start_pos, snap)


def run_c(q, k, v, g, beta, s0=None, scale=None, start_pos=0, snap=0):
    return native.oracle_sequence(q, k, v, g, beta, s0, scale, start_pos, snap)


def make_chunked(C):
    def run(q, k, v, g, beta, s0=None, scale=None, start_pos=0, snap=0):
        ok = snap > 0 and snap % C == 0 and start_pos % C == 0
        o, S, sn = kda_chunked(q, k, v, g, beta, s0, scale, C, start_pos, snap if ok else 0)
        return o, S, (sn if ok or snap == 0 else None)
    return run


IMPLS = {"numpy": run_numpy, "c": run_c, "chunk4": make_chunked(4),
         "chunk16": make_chunked(16), "chunk64": make_chunked(64)}
# fp32-input implementations see inputs rounded to fp32 (the C oracle's input
# type); where a pin's inputs are not fp32-exact its tolerance says so.
FP32_INPUT = {"c"}


def _rand(seed, T, H, d, fp32=True):
    x = synth.token_inputs(seed, T, H, d, d, io="fp32")
    return {kk: vv.numpy().astype(np.float64) for kk, vv in x.items()}


# --------------------------------------------------------------------------
# pins, written as checks that raise AssertionError
# --------------------------------------------------------------------------
def pin_exact_product(run, name):
    """Exact rational product form (tests/golden/exact_product_T8_d4.json)."""
    data = json.loads(GOLDEN.read_text())
    for case in data["cases"]:
        fr = lambda m: np.array([[float(Fraction(x)) for x in row] for row in m])
        q, k, v, a, s0 = (fr(case[n]) for n in ("q", "k", "v", "alpha", "s0"))
        beta = np.array([float(Fraction(x)) for x in case["beta"]])
        g = np.log(a)
        T = case["T"]
        o, S, sn = run(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None],
                       s0[None], 0.5, 0, 1)
        o_ref = fr(case["o"])
        st_ref = np.stack([fr(m) for m in case["states"]])
        # g = log(alpha) is rounded to fp64 (or fp32 for the C oracle's input);
        # over 8 tokens that perturbs the decays by < 8 * 2^-24 * max|g| < 1e-6.
        tol = 2e-6 if name in FP32_INPUT else 1e-13
        assert normwise_rel_err(o[:, 0], o_ref) <= tol, (case["name"], "o")
        assert normwise_rel_err(S[0], st_ref[-1]) <= tol, (case["name"], "S_T")
        if sn is not None:
            assert sn.shape[0] == st_ref.shape[0], (case["name"], "snapshot count")
            assert normwise_rel_err(sn[:, 0], st_ref) <= tol, (case["name"], "S_t")


def pin_beta_zero(run, name):
    """beta = 0: S_t = Diag(Gamma_t) S_0, o_t = scale * S_0^T (Gamma_t . q_t)."""
    x = _rand(11, 40, 3, 16)
    s0 = synth.states(11, 1, 3, 16, 16, std=1.0)[0].numpy().astype(np.float64)
    beta = np.zeros_like(x["beta"])
    o, S, _ = run(x["q"], x["k"], x["v"], x["g"], beta, s0, 0.25)
    Gam = np.exp(np.cumsum(x["g"], axis=0))                   # [T, H, dk]
    o_ref = 0.25 * np.einsum("thi,hij->thj", Gam * x["q"], s0)
    S_ref = Gam[-1][:, :, None] * s0
    assert normwise_rel_err(o, o_ref) <= 1e-12
    assert normwise_rel_err(S, S_ref) <= 1e-12


def pin_orthogonal_keys(run, name):
    """Distinct basis-vector keys, S_0 = 0: the erase term vanishes and KDA is
    decayed linear attention, o_t = scale sum_{i<=t} beta_i q_{t,c_i}
    prod_{i<j<=t} alpha_{j,c_i} v_i."""
    T, H, d = 24, 2, 32
    x = _rand(12, T, H, d)
    order = synth.permutation(12, d)[:T]
    k = np.zeros((T, H, d))
    for t in range(T):
        k[t, :, order[t]] = 1.0
    o, S, _ = run(x["q"], k, x["v"], x["g"], x["beta"], None, 0.5)
    b = np.cumsum(x["g"], axis=0)
    o_ref = np.zeros((T, H, d))
    for t in range(T):
        for i in range(t + 1):
            c = order[i]
            w = x["beta"][i] * x["q"][t, :, c] * np.exp(b[t, :, c] - b[i, :, c])
            o_ref[t] += 0.5 * w[:, None] * x["v"][i]
    assert normwise_rel_err(o, o_ref) <= 1e-12


def pin_overwrite(run, name):
    """alpha = 1, beta = 1, orthonormal keys: reading with q = k_j returns the
    value of the latest write to k_j (times scale); repeated keys replace."""
    T, d = 30, 16
    rng = np.random.default_rng(13)
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    basis = Qm.T[:6]
    if name in FP32_INPUT:
        basis = basis.astype(np.float32).astype(np.float64)
    key_ids = rng.integers(0, 6, size=T)
    v = rng.standard_normal((T, 1, d))
    k = basis[key_ids][:, None, :]
    q = np.zeros_like(k)
    expect = np.zeros((T, 1, d))
    last = {}
    for t in range(T):
        last[key_ids[t]] = v[t, 0]
        j = rng.choice(sorted(last))
        q[t, 0] = basis[j]
        expect[t, 0] = 0.25 * last[j]
    g = np.zeros((T, 1, d))
    beta = np.ones((T, 1))
    o, _, _ = run(q, k, v, g, beta, None, 0.25)
    tol = 1e-5 if name in FP32_INPUT else 1e-12
    assert normwise_rel_err(o, expect) <= tol


def pin_unit_key_read(run, name):
    """beta_t = 1 and |k_t| = 1 give S_t^T k_t = v_t exactly, for any gate and
    any previous state: with q_t = k_t, o_t = scale * v_t."""
    x = _rand(14, 50, 2, 16)
    s0 = synth.states(14, 1, 2, 16, 16, std=1.0)[0].numpy().astype(np.float64)
    k = x["k"] / np.linalg.norm(x["k"], axis=-1, keepdims=True)
    if name in FP32_INPUT:
        k = k.astype(np.float32).astype(np.float64)
    beta = np.ones_like(x["beta"])
    o, _, _ = run(k, k, x["v"], x["g"], beta, s0, 0.25)
    tol = 1e-5 if name in FP32_INPUT else 1e-12
    assert normwise_rel_err(o, 0.25 * x["v"]) <= tol


def pin_linearity(run, name):
    """o and S are jointly linear in (S_0, V) for fixed q, k, g, beta."""
    x = _rand(15, 37, 2, 16)
    sa = synth.states(15, 2, 2, 16, 16, std=1.0).numpy().astype(np.float64)
    vb = synth.token_inputs(16, 37, 2, 16, 16, io="fp32")["v"].numpy().astype(np.float64)
    c = 0.75
    oa, Sa, _ = run(x["q"], x["k"], x["v"], x["g"], x["beta"], sa[0])
    ob, Sb, _ = run(x["q"], x["k"], vb, x["g"], x["beta"], sa[1])
    oc, Sc, _ = run(x["q"], x["k"], x["v"] + c * vb, x["g"], x["beta"], sa[0] + c * sa[1])
    # the combined inputs are rounded to fp32 on the way into the C oracle
    tol = 1e-6 if name in FP32_INPUT else 1e-12
    assert normwise_rel_err(oc, oa + c * ob) <= tol
    assert normwise_rel_err(Sc, Sa + c * Sb) <= tol


def pin_permutation(run, name):
    """d_v columns and heads are independent: permuting v's columns permutes the
    columns of o and S; permuting heads permutes the outputs."""
    x = _rand(17, 33, 3, 16)
    s0 = synth.states(17, 1, 3, 16, 16, std=1.0)[0].numpy().astype(np.float64)
    perm = np.array(synth.permutation(17, 16))
    hp = np.array([2, 0, 1])
    o, S, _ = run(x["q"], x["k"], x["v"], x["g"], x["beta"], s0)
    o2, S2, _ = run(x["q"], x["k"], x["v"][:, :, perm], x["g"], x["beta"], s0[:, :, perm])
    assert normwise_rel_err(o2, o[:, :, perm]) <= 1e-14
    assert normwise_rel_err(S2, S[:, :, perm]) <= 1e-14
    o3, S3, _ = run(x["q"][:, hp], x["k"][:, hp], x["v"][:, hp], x["g"][:, hp],
                    x["beta"][:, hp], s0[hp])
    assert normwise_rel_err(o3, o[:, hp]) <= 1e-14
    assert normwise_rel_err(S3, S[hp]) <= 1e-14


def pin_bounded(run, name):
    """|k| = 1 and beta in [0, 1] make (I - beta k k^T) Diag(alpha) a
    contraction, so |S_t|_2 <= |S_{t-1}|_2 + beta_t |v_t| (spectral norms)."""
    x = _rand(18, 64, 2, 16)
    s0 = synth.states(18, 1, 2, 16, 16, std=1.0)[0].numpy().astype(np.float64)
    interval = int(name[5:]) if name.startswith("chunk") else 1
    o, S, sn = run(x["q"], x["k"], x["v"], x["g"], x["beta"], s0, None, 0, interval)
    assert sn is not None and len(sn) == 64 // interval
    prev = s0
    vn = np.linalg.norm(x["v"], axis=-1) * x["beta"]          # [T, H]
    for j in range(len(sn)):
        lo, hi = j * interval, (j + 1) * interval
        for h in range(2):
            grow = np.linalg.norm(sn[j, h], 2) - np.linalg.norm(prev[h], 2)
            assert grow <= vn[lo:hi, h].sum() + 1e-12
        prev = sn[j]


def pin_token_equals_reference_loop(run, name):
    """Snapshots and outputs of every implementation agree with the plain numpy
    token loop on random inputs, with a start position and ragged length."""
    x = _rand(19, 150, 2, 16)
    s0 = synth.states(19, 1, 2, 16, 16, std=1.0)[0].numpy().astype(np.float64)
    ref = kda_recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], s0, None, 64, 32)
    got = run(x["q"], x["k"], x["v"], x["g"], x["beta"], s0, None, 64, 32)
    assert normwise_rel_err(got[0], ref[0]) <= 1e-12
    assert normwise_rel_err(got[1], ref[1]) <= 1e-12
    if got[2] is not None:
        assert got[2].shape == ref[2].shape
        assert normwise_rel_err(got[2], ref[2]) <= 1e-12


PINS = [pin_exact_product, pin_beta_zero, pin_orthogonal_keys, pin_overwrite,
        pin_unit_key_read, pin_linearity, pin_permutation, pin_bounded]


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin, impl):
    pin(IMPLS[impl], impl)


@pytest.mark.parametrize("impl", ["c", "chunk4", "chunk16", "chunk64"])
def test_agrees_with_numpy_token_loop(impl):
    pin_token_equals_reference_loop(IMPLS[impl], impl)


@pytest.mark.parametrize("C", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 200])
def test_chunked_equals_token(C, T):
    """The derived chunk algebra equals the token recurrence (<= 1e-12) for
    lengths that are and are not multiples of the chunk, with snapshots."""
    x = _rand(20 + T, T, 2, 32)
    s0 = synth.states(20, 1, 2, 32, 32, std=1.0)[0].numpy().astype(np.float64)
    start = 2 * C
    ref = kda_recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], s0, None, start, 2 * C)
    got = kda_chunked(x["q"], x["k"], x["v"], x["g"], x["beta"], s0, None, C, start, 2 * C)
    assert normwise_rel_err(got[0], ref[0]) <= 1e-12
    assert normwise_rel_err(got[1], ref[1]) <= 1e-12
    assert got[2].shape == ref[2].shape
    if len(ref[2]):
        assert normwise_rel_err(got[2], ref[2]) <= 1e-12


@pytest.mark.parametrize("impl", ["numpy", "c"])
def test_resume_from_snapshot_is_bit_identical(impl):
    """Resuming from the oracle's own snapshot at position p reproduces the full
    run exactly: same operations in the same order."""
    run = IMPLS[impl]
    x = _rand(21, 300, 2, 16)
    o, S, sn = run(x["q"], x["k"], x["v"], x["g"], x["beta"], None, None, 0, 64)
    for m in range(len(sn)):
        p = 64 * (m + 1)
        o2, S2, sn2 = run(*(x[n][p:] for n in ("q", "k", "v", "g", "beta")), sn[m], None, p, 64)
        assert np.array_equal(o2, o[p:])
        assert np.array_equal(S2, S)
        assert np.array_equal(sn2, sn[m + 1:])


@pytest.mark.parametrize("start,length,interval", [
    (0, 0, 256), (0, 255, 256), (0, 256, 256), (0, 257, 256), (256, 256, 256),
    (512, 1000, 256), (4096, 65536, 4096), (7, 100, 16), (0, 100, 0), (3, 1, 4)])
def test_snapshot_rule(start, length, interval):
    """Snapshot positions are the multiples of the interval in
    (start, start + length], ascending; brute-force enumeration agrees."""
    brute = [p for p in range(start + 1, start + length + 1) if interval and p % interval == 0]
    assert snapshot_positions(start, length, interval) == brute
    assert snapshot_count(start, length, interval) == len(brute)


def test_exact_fixture_is_reproducible():
    """The stored exact fixture is what oracle/exact.py computes today."""
    from oracle.exact import kda_exact
    data = json.loads(GOLDEN.read_text())
    for case in data["cases"]:
        fr = lambda m: [[Fraction(x) for x in row] for row in m]
        o, S = kda_exact(fr(case["q"]), fr(case["k"]), fr(case["v"]), fr(case["alpha"]),
                         [Fraction(b) for b in case["beta"]], fr(case["s0"]), Fraction(1, 2))
        assert [[f"{x.numerator}/{x.denominator}" for x in r] for r in o] == case["o"]
        assert [[[f"{x.numerator}/{x.denominator}" for x in r] for r in m] for m in S] == case["states"]


# --------------------------------------------------------------------------
# planted mistakes: each mutant of the token loop must fail at least one pin
# --------------------------------------------------------------------------
def _mutant(kind):
    def run(q, k, v, g, beta, s0=None, scale=None, start_pos=0, snap=0):
        q, k, v, g, beta = (np.asarray(a, dtype=np.float64) for a in (q, k, v, g, beta))
        T, H, dk = k.shape
        dv = v.shape[2]
        scale = 1.0 / np.sqrt(dk) if scale is None else scale
        S = np.zeros((H, dk, dv)) if s0 is None else np.array(s0, dtype=np.float64)
        o = np.zeros((T, H, dv))
        snaps = []
        for t in range(T):
            a = np.exp(g[t])
            if kind != "gate_after_delta":
                S = (a[:, None, :] if kind == "gate_on_value_axis" else a[:, :, None]) * S
            x = np.einsum("hij,hi->hj", S, k[t])
            if kind == "erase_sign":
                x = -x
            if kind == "drop_erase":
                x = 0 * x
            S_prev = S
            S = S + beta[t][:, None, None] * k[t][:, :, None] * (v[t] - x)[:, None, :]
            if kind == "gate_after_delta":
                S = a[:, :, None] * S
            read = S_prev if kind == "read_before_update" else S
            if kind == "transposed_read":
                o[t] = scale * np.einsum("hij,hj->hi", read, q[t])
            else:
                o[t] = scale * np.einsum("hij,hi->hj", read, q[t])
            if kind == "no_scale":
                o[t] /= scale
            p = start_pos + t + 1
            if snap > 0 and p % snap == (1 if kind == "snapshot_off_by_one" else 0):
                snaps.append(S.copy())
        return o, S, (np.stack(snaps) if snaps else np.zeros((0, H, dk, dv)))
    return run


MUTANTS = ["gate_after_delta", "gate_on_value_axis", "erase_sign", "drop_erase",
           "read_before_update", "transposed_read", "no_scale", "snapshot_off_by_one"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_mistake_is_caught(kind):
    run = _mutant(kind)
    caught = []
    for pin in PINS:
        try:
            pin(run, "mutant")
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {kind}"
