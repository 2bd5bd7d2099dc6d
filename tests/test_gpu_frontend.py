"""GPU parity of the q/k front-end (short causal conv, Swish, L2 normalisation;
Kimi K3 technical FAQ, "What is KDA") through the C ABI, against oracle/frontend.py
followed by the fp64 token recurrence (oracle/native.py):

  kda_qk_frontend          ragged packed batches with carried conv states and
                           block-boundary conv snapshots;
  kda_qk_frontend + prefill the whole prefill pipeline, on all three prefill paths,
                           including resume from a snapshot of both states;
  kda_decode_conv, kda_verify_conv, kda_verify_commit_conv
                           the front-end fused into the token loads.

The oracle's normalised features are rounded by the oracle itself to the I/O type
before its recurrence where the interface hands them over in that type
(kda_qk_frontend's q_out, k_out); the decode-side kernels keep them in fp32 and the
oracle does not round. Conv states hold raw inputs and are compared exactly.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from hybrid_linear_attention_04_b200 import kda as K
from kda_cases import TOL_BF16, TOL_FP32, check_outputs, check_states, to_np, tol_for
from oracle import frontend as F
from oracle import native

pytestmark = pytest.mark.gpu


def _io_round(x, io):
    """Round fp64 features to the I/O type (RNE), as the interface hands them over."""
    t = torch.from_numpy(np.ascontiguousarray(x)).float()
    return (t.to(torch.bfloat16) if io == "bf16" else t).double().numpy()


def _oracle_frontend(raw, cu, wq, wk, conv_in, start, snap):
    """(features q, k [T, H, d], final conv states [n, 2, H, d, K-1], snapshots)."""
    ci_q = None if conv_in is None else conv_in[:, 0].double().numpy()
    ci_k = None if conv_in is None else conv_in[:, 1].double().numpy()
    fq, sq, snq = F.qk_frontend_packed(raw["q"].double().numpy(), cu, wq.double().numpy(), ci_q,
                                       start, snap)
    fk, sk, snk = F.qk_frontend_packed(raw["k"].double().numpy(), cu, wk.double().numpy(), ci_k,
                                       start, snap)
    return fq, fk, np.stack([sq, sk], axis=1), np.stack([snq, snk], axis=1)


def _gpu_frontend(raw_d, cu, wq_d, wk_d, conv_in_d, start, snap, chunk, H, d):
    T, n = int(cu[-1]), len(cu) - 1
    taps = wq_d.shape[-1]
    qo = torch.empty_like(raw_d["q"])
    ko = torch.empty_like(raw_d["k"])
    co = torch.full((n, 2, H, d, taps - 1), float("nan"), device=qo.device)
    offs, _ = K.kda_snapshot_plan(cu, start, snap)
    csn = torch.full((int(offs[-1]) + 1, 2, H, d, taps - 1), float("nan"), device=qo.device)
    K.kda_qk_frontend(raw_d["q"], raw_d["k"], wq_d, wk_d, cu, qo, ko, conv_in=conv_in_d,
                      conv_out=co, start_pos=start, snap_interval=snap, conv_snapshots=csn,
                      chunk=chunk)
    assert K.kda_check_device_status() == 0
    assert torch.isnan(csn[int(offs[-1])]).all()
    return qo, ko, co, csn[:int(offs[-1])]


@pytest.mark.parametrize("d,chunk,io,taps", [(128, 64, "bf16", 4), (64, 32, "fp32", 2),
                                             (32, 16, "bf16", 3), (128, 16, "fp32", 4)])
def test_frontend_matches_oracle(cuda_device, d, chunk, io, taps):
    lens = [0, 1, 2, chunk - 1, chunk, 3 * chunk + 5, 7 * chunk]
    H, n = 3, len(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    raw = synth.raw_qk(500 + taps, int(cu[-1]), H, d, io=io)
    wq, wk = synth.conv_weights(501, H, d, taps)
    conv_in = synth.conv_states(502, n, H, d, taps, io=io)
    start = [chunk * m for m in (0, 1, 3, 2, 0, 1, 5)]
    snap = 2 * chunk
    dev = lambda t: t.to(cuda_device)  # noqa: E731
    qo, ko, co, csn = _gpu_frontend({k: dev(v) for k, v in raw.items()}, cu, dev(wq), dev(wk),
                                    dev(conv_in), start, snap, chunk, H, d)
    fq, fk, cs, sn = _oracle_frontend(raw, cu, wq, wk, conv_in, start, snap)
    tol = tol_for(io)
    check_outputs("q features", to_np(qo), fq, tol, cu)
    check_outputs("k features", to_np(ko), fk, tol, cu)
    assert np.array_equal(co.cpu().double().numpy(), cs)          # raw inputs, exactly
    assert csn.shape[0] == sn.shape[0] and np.array_equal(csn.cpu().double().numpy(), sn)


_PATHS = {"split": (0, "auto"), "fused": (0, None), "simt": (1, "auto")}


@pytest.mark.parametrize("path", ["split", "fused", "simt"])
def test_frontend_then_prefill_matches_oracle_pipeline(cuda_device, path):
    """Raw q, k through kda_qk_frontend then kda_prefill (ragged, initial states and
    conv states, snapshots) against the oracle front-end followed by the fp64 token
    recurrence."""
    d, chunk, H, taps = 128, 64, 4, 4
    lens = [300, 64, 0, 129, 5]
    n = len(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    x = synth.token_inputs(520, T, H, d, d, io="bf16")
    raw = synth.raw_qk(520, T, H, d, io="bf16")
    wq, wk = synth.conv_weights(521, H, d, taps)
    conv_in = synth.conv_states(522, n, H, d, taps)
    s0 = synth.states(523, n, H, d, d, std=0.1)
    start = [0, 128, 64, 256, 0]
    snap = 128
    dev = lambda t: t.to(cuda_device)  # noqa: E731
    qo, ko, co, csn = _gpu_frontend({k: dev(v) for k, v in raw.items()}, cu, dev(wq), dev(wk),
                                    dev(conv_in), start, snap, chunk, H, d)
    force, ws = _PATHS[path]
    K.lib().kda_internal_force_prefill_path(force)
    try:
        o = torch.empty((T, H, d), dtype=torch.bfloat16, device=cuda_device)
        so = torch.empty((n, H, d, d), device=cuda_device)
        offs, _ = K.kda_snapshot_plan(cu, start, snap)
        sn = torch.empty((int(offs[-1]), H, d, d), device=cuda_device)
        K.kda_prefill(qo, ko, dev(x["v"]), dev(x["g"]), dev(x["beta"]), cu, o, state_out=so,
                      state_in=dev(s0), start_pos=start, snap_interval=snap, snapshots=sn,
                      chunk=chunk, workspace=ws)
        assert K.kda_check_device_status() == 0
    finally:
        K.lib().kda_internal_force_prefill_path(0)
    fq, fk, _, _ = _oracle_frontend(raw, cu, wq, wk, conv_in, start, snap)
    o_ref, s_ref, sn_ref = native.oracle_packed(_io_round(fq, "bf16"), _io_round(fk, "bf16"),
                                                x["v"], x["g"], x["beta"], cu, start, s0, None,
                                                snap)
    check_outputs("o", to_np(o), o_ref, TOL_BF16, cu)
    check_states("state", to_np(so), s_ref, TOL_BF16, (2, 3))
    check_states("snapshots", sn.cpu().numpy(), sn_ref, TOL_BF16, (2, 3))


def test_frontend_resume_from_conv_snapshot_equals_full_run(cuda_device):
    """Prefix caching with the front-end: a sequence resumed from its own block-boundary
    conv snapshot gives the same features, bit for bit, as the uninterrupted run."""
    d, chunk, H, taps, T, snap = 128, 64, 2, 4, 600, 128
    raw = synth.raw_qk(530, T, H, d, io="bf16")
    wq, wk = synth.conv_weights(531, H, d, taps)
    dev = lambda t: t.to(cuda_device)  # noqa: E731
    raw_d = {k: dev(v) for k, v in raw.items()}
    cu = np.array([0, T], dtype=np.int32)
    qo, ko, co, csn = _gpu_frontend(raw_d, cu, dev(wq), dev(wk), None, None, snap, chunk, H, d)
    for m in range(csn.shape[0]):
        p = snap * (m + 1)
        sub = {k: v[p:].contiguous() for k, v in raw_d.items()}
        q2, k2, c2, _ = _gpu_frontend(sub, np.array([0, T - p], dtype=np.int32), dev(wq), dev(wk),
                                      csn[m:m + 1].contiguous(), [p], snap, chunk, H, d)
        assert torch.equal(q2, qo[p:]) and torch.equal(k2, ko[p:]) and torch.equal(c2, co)


def _decode_conv_case(seed, n_seq, H, d, io, taps, device):
    x = synth.token_inputs(seed, n_seq, H, d, d, io=io)
    raw = synth.raw_qk(seed, n_seq, H, d, io=io)
    pool = synth.states(seed, n_seq + 2, H, d, d, std=0.1)
    cpool = synth.conv_states(seed, n_seq + 2, H, d, taps, io=io)
    wq, wk = synth.conv_weights(seed, H, d, taps)
    slots = synth.permutation(seed, n_seq + 2, "slots")[:n_seq]
    return x, raw, pool, cpool, wq, wk, slots


@pytest.mark.parametrize("d,io,H,n_seq,taps", [(128, "bf16", 64, 512, 4), (64, "fp32", 3, 9, 3),
                                               (32, "bf16", 2, 5, 2)])
def test_decode_conv_matches_oracle(cuda_device, d, io, H, n_seq, taps):
    x, raw, pool, cpool, wq, wk, slots = _decode_conv_case(600 + d, n_seq, H, d, io, taps, cuda_device)
    dev = lambda t: t.to(cuda_device)  # noqa: E731
    pool_d, cpool_d = dev(pool), dev(cpool)
    o = torch.empty((n_seq, H, d), dtype=x["v"].dtype, device=cuda_device)
    K.kda_decode_conv(dev(raw["q"]), dev(raw["k"]), dev(x["v"]), dev(x["g"]), dev(x["beta"]),
                      torch.tensor(slots, dtype=torch.int32, device=cuda_device), pool_d, cpool_d,
                      o, dev(wq), dev(wk))
    assert K.kda_check_device_status() == 0
    o_ref = np.zeros((n_seq, H, d))
    s_ref, c_ref = [], []
    for s in range(n_seq):
        sl = slots[s]
        fq, _ = F.qk_frontend(raw["q"][s:s + 1].double().numpy(), wq.double().numpy(),
                              cpool[sl, 0].double().numpy())
        fk, nk = F.qk_frontend(raw["k"][s:s + 1].double().numpy(), wk.double().numpy(),
                               cpool[sl, 1].double().numpy())
        _, nq = F.short_conv(raw["q"][s:s + 1].double().numpy(), wq.double().numpy(),
                             cpool[sl, 0].double().numpy())
        oo, st, _ = native.oracle_sequence(fq, fk, x["v"][s:s + 1], x["g"][s:s + 1],
                                           x["beta"][s:s + 1], pool[sl])
        o_ref[s] = oo[0]
        s_ref.append(st)
        c_ref.append(np.stack([nq, nk]))
    tol = TOL_BF16 if io == "bf16" else TOL_FP32
    check_outputs("o", to_np(o), o_ref, tol, np.arange(n_seq + 1))
    check_states("state", to_np(pool_d)[slots], np.stack(s_ref), tol, (2, 3))
    assert np.array_equal(cpool_d.cpu().double().numpy()[slots], np.stack(c_ref))


def _verify_conv_case(seed, n_seq, H, d, io, taps, device):
    lens = synth.draft_lengths(seed, n_seq, 1, 8)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    x = synth.token_inputs(seed, T, H, d, d, io=io)
    raw = synth.raw_qk(seed, T, H, d, io=io)
    pool = synth.states(seed, n_seq + 2, H, d, d, std=0.1)
    cpool = synth.conv_states(seed, n_seq + 2, H, d, taps, io=io)
    wq, wk = synth.conv_weights(seed, H, d, taps)
    slots = synth.permutation(seed, n_seq + 2, "slots")[:n_seq]
    dev = lambda t: t.to(device)  # noqa: E731
    return dict(cu=cu, x=x, raw=raw, pool=pool, cpool=cpool, wq=wq, wk=wk, slots=slots,
                xd={k: dev(v) for k, v in x.items()}, rd={k: dev(v) for k, v in raw.items()},
                wqd=dev(wq), wkd=dev(wk), slots_d=torch.tensor(slots, dtype=torch.int32, device=device))


@pytest.mark.parametrize("d,io,H,n_seq,taps", [(128, "bf16", 16, 64, 4), (64, "fp32", 2, 7, 2)])
def test_verify_conv_matches_oracle(cuda_device, d, io, H, n_seq, taps):
    c = _verify_conv_case(610 + d, n_seq, H, d, io, taps, cuda_device)
    cu, x, raw = c["cu"], c["x"], c["raw"]
    T = int(cu[-1])
    pool_d, cpool_d = c["pool"].to(cuda_device), c["cpool"].to(cuda_device)
    ts = torch.empty((T, H, d, d), device=cuda_device)
    cts = torch.empty((T, 2, H, d, taps - 1), device=cuda_device)
    o = torch.empty((T, H, d), dtype=x["v"].dtype, device=cuda_device)
    K.kda_verify_conv(c["rd"]["q"], c["rd"]["k"], c["xd"]["v"], c["xd"]["g"], c["xd"]["beta"], cu,
                      c["slots_d"], pool_d, cpool_d, ts, o, c["wqd"], c["wkd"],
                      conv_token_states=cts)
    assert K.kda_check_device_status() == 0
    assert torch.equal(cpool_d.cpu(), c["cpool"]) and torch.equal(pool_d.cpu(), c["pool"])
    tol = TOL_BF16 if io == "bf16" else TOL_FP32
    o_ref, ts_ref = np.zeros((T, H, d)), np.zeros((T, H, d, d))
    cts_got = cts.cpu().double().numpy()
    for s in range(n_seq):
        a, b, sl = int(cu[s]), int(cu[s + 1]), c["slots"][s]
        wq64, wk64 = c["wq"].double().numpy(), c["wk"].double().numpy()
        fq, _ = F.qk_frontend(raw["q"][a:b].double().numpy(), wq64, c["cpool"][sl, 0].double().numpy())
        fk, _ = F.qk_frontend(raw["k"][a:b].double().numpy(), wk64, c["cpool"][sl, 1].double().numpy())
        oo, _, sn = native.oracle_sequence(fq, fk, x["v"][a:b], x["g"][a:b], x["beta"][a:b],
                                           c["pool"][sl], None, 0, 1)
        o_ref[a:b], ts_ref[a:b] = oo, sn
        for j in range(b - a):
            _, nq = F.short_conv(raw["q"][a:a + j + 1].double().numpy(), wq64,
                                 c["cpool"][sl, 0].double().numpy())
            _, nk = F.short_conv(raw["k"][a:a + j + 1].double().numpy(), wk64,
                                 c["cpool"][sl, 1].double().numpy())
            assert np.array_equal(cts_got[a + j], np.stack([nq, nk])), (s, j)
    check_outputs("o", to_np(o), o_ref, tol, cu)
    check_states("token states", ts.cpu().numpy(), ts_ref, tol, (2, 3))


def test_verify_commit_conv_bit_identical_to_verify_conv_and_snapshot(cuda_device):
    """The fused step with the front-end equals kda_verify_conv of the previous batch,
    kda_snapshot commits of both the recurrent and the conv state of the accepted token,
    then kda_verify_conv of this batch: states, conv states and outputs bit for bit; the
    block-boundary snapshot pair equals the per-token states there."""
    H, d, n_seq, taps, snap = 8, 128, 32, 4, 64
    c = _verify_conv_case(640, n_seq, H, d, "bf16", taps, cuda_device)
    nxt = _verify_conv_case(641, n_seq, H, d, "bf16", taps, cuda_device)
    cp, cd = c["cu"], nxt["cu"]
    acc = [min(a, int(cp[s + 1] - cp[s])) for s, a in enumerate(synth.randint(640, "misc", n_seq, 0, 8))]
    pos = [snap * (s + 1) - 1 - (s % 6) for s in range(n_seq)]
    pool_a, cpool_a = c["pool"].to(cuda_device), c["cpool"].to(cuda_device)
    pool_b, cpool_b = pool_a.clone(), cpool_a.clone()
    # reference: verify with per-token states, commit both states, verify the next batch
    Tp = int(cp[-1])
    ts = torch.empty((Tp, H, d, d), device=cuda_device)
    cts = torch.empty((Tp, 2, H, d, taps - 1), device=cuda_device)
    op = torch.empty((Tp, H, d), dtype=torch.bfloat16, device=cuda_device)
    K.kda_verify_conv(c["rd"]["q"], c["rd"]["k"], c["xd"]["v"], c["xd"]["g"], c["xd"]["beta"], cp,
                      c["slots_d"], pool_a, cpool_a, ts, op, c["wqd"], c["wkd"], conv_token_states=cts)
    keep = [s for s in range(n_seq) if acc[s] > 0]
    src = torch.tensor([int(cp[s]) + acc[s] - 1 for s in keep], dtype=torch.int64, device=cuda_device)
    dst = torch.tensor([c["slots"][s] for s in keep], dtype=torch.int64, device=cuda_device)
    K.kda_snapshot(src, dst, ts, pool_a)
    K.kda_snapshot(src, dst, cts.view(Tp, 2 * H, d, taps - 1), cpool_a.view(-1, 2 * H, d, taps - 1))
    Tc = int(cd[-1])
    ts2 = torch.empty((Tc, H, d, d), device=cuda_device)
    o_ref = torch.empty((Tc, H, d), dtype=torch.bfloat16, device=cuda_device)
    K.kda_verify_conv(nxt["rd"]["q"], nxt["rd"]["k"], nxt["xd"]["v"], nxt["xd"]["g"], nxt["xd"]["beta"],
                      cd, c["slots_d"], pool_a, cpool_a, ts2, o_ref, c["wqd"], c["wkd"])
    # fused, with a snapshot row per sequence
    sn = torch.full((n_seq, H, d, d), float("nan"), device=cuda_device)
    csn = torch.full((n_seq, 2, H, d, taps - 1), float("nan"), device=cuda_device)
    prev = {"q": c["rd"]["q"], "k": c["rd"]["k"], "v": c["xd"]["v"], "g": c["xd"]["g"],
            "beta": c["xd"]["beta"]}
    o = torch.empty((Tc, H, d), dtype=torch.bfloat16, device=cuda_device)
    K.kda_verify_commit_conv(prev, torch.tensor(acc, dtype=torch.int32, device=cuda_device), cp,
                             nxt["rd"]["q"], nxt["rd"]["k"], nxt["xd"]["v"], nxt["xd"]["g"],
                             nxt["xd"]["beta"], cd, c["slots_d"], pool_b, cpool_b, o, c["wqd"],
                             c["wkd"], pos=torch.tensor(pos, dtype=torch.int64, device=cuda_device),
                             snap_interval=snap,
                             snap_row=torch.arange(n_seq, dtype=torch.int64, device=cuda_device),
                             snapshots=sn, conv_snapshots=csn)
    assert K.kda_check_device_status() == 0
    assert torch.equal(pool_a, pool_b) and torch.equal(cpool_a, cpool_b) and torch.equal(o, o_ref)
    crossed = 0
    for s in range(n_seq):
        j = snap * (pos[s] // snap + 1) - pos[s] - 1
        if j < acc[s]:
            assert torch.equal(sn[s], ts[int(cp[s]) + j]) and torch.equal(csn[s], cts[int(cp[s]) + j])
            crossed += 1
        else:
            assert torch.isnan(sn[s]).all() and torch.isnan(csn[s]).all()
    assert 0 < crossed < n_seq
