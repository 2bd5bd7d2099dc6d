"""GPU parity of kda_verify_commit (a speculative step with the previous step's
commit fused in) against the fp64 oracle and against kda_verify + kda_snapshot,
through the C ABI.

The oracle runs, per sequence, the previous batch's accepted prefix followed by
this step's drafts from the slot's state (token recurrence; Kimi K3 technical
FAQ, "What is KDA"): the committed state is its state after the prefix, and the
outputs are its outputs for the drafts. Acceptance counts are seeded (uniform in
0..m for a previous batch of m tokens; runtimewire, "A third party tripled
single-user decoding speed": a prefix of each step's drafts is accepted).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from hybrid_linear_attention_04_b200 import kda as K
from kda_cases import TOL_BF16, TOL_FP32, check_outputs, check_states, same_outputs, same_states, to_np
from oracle import native

pytestmark = pytest.mark.gpu


def _case(seed, n_seq, H, d, io, device, lo=1, hi=8):
    lp = synth.draft_lengths(seed, n_seq, lo, hi)
    lc = synth.draft_lengths(seed + 1, n_seq, lo, hi)
    cp = np.concatenate([[0], np.cumsum(lp)]).astype(np.int32)
    cd = np.concatenate([[0], np.cumsum(lc)]).astype(np.int32)
    xp = synth.token_inputs(seed, int(cp[-1]), H, d, d, io=io)
    xc = synth.token_inputs(seed + 1, int(cd[-1]), H, d, d, io=io)
    acc = [min(a, m) for a, m in zip(synth.randint(seed, "misc", n_seq, 0, 8), lp)]
    pool = synth.states(seed, n_seq + 3, H, d, d, std=0.1)
    slots = synth.permutation(seed, n_seq + 3, "slots")[:n_seq]
    dev = lambda x: {k: v.to(device) for k, v in x.items()}  # noqa: E731
    return dict(cp=cp, cd=cd, xp=xp, xc=xc, dp=dev(xp), dc=dev(xc), acc=acc, pool=pool,
                slots=slots, n_seq=n_seq, H=H, d=d,
                acc_d=torch.tensor(acc, dtype=torch.int32, device=device),
                slots_d=torch.tensor(slots, dtype=torch.int32, device=device))


def _fused(c, pool_d, **kw):
    o = torch.empty((int(c["cd"][-1]), c["H"], c["d"]), dtype=c["dc"]["v"].dtype,
                    device=pool_d.device)
    dc = c["dc"]
    K.kda_verify_commit(c["dp"], c["acc_d"], c["cp"], dc["q"], dc["k"], dc["v"], dc["g"],
                        dc["beta"], c["cd"], c["slots_d"], pool_d, o, **kw)
    return o


@pytest.mark.parametrize("d,io,H,n_seq", [(128, "bf16", 64, 512), (128, "fp32", 2, 9),
                                          (64, "bf16", 3, 17), (32, "fp32", 2, 6)])
def test_verify_commit_matches_oracle(cuda_device, d, io, H, n_seq):
    c = _case(700 + d, n_seq, H, d, io, cuda_device)
    pool_d = c["pool"].to(cuda_device)
    o = _fused(c, pool_d)
    assert K.kda_check_device_status() == 0
    tol = TOL_BF16 if io == "bf16" else TOL_FP32
    got_pool, got_o = pool_d.cpu(), to_np(o)
    o_ref = np.zeros_like(got_o)
    s_ref, s_got = [], []
    xp, xc, cp, cd = c["xp"], c["xc"], c["cp"], c["cd"]
    for s in range(n_seq):
        a, na = int(cp[s]), c["acc"][s]
        b0, b1 = int(cd[s]), int(cd[s + 1])
        seq = {k: torch.cat([xp[k][a:a + na], xc[k][b0:b1]]) for k in xp}
        oo, _, sn = native.oracle_sequence(seq["q"], seq["k"], seq["v"], seq["g"], seq["beta"],
                                           c["pool"][c["slots"][s]], None, 0, 1)
        o_ref[b0:b1] = oo[na:]
        slot = c["slots"][s]
        if na == 0:
            assert torch.equal(got_pool[slot], c["pool"][slot])      # not written
        else:
            s_ref.append(sn[na - 1])
            s_got.append(got_pool[slot].double().numpy())
    check_outputs("o", got_o, o_ref, tol, cd)
    check_states("committed state", np.stack(s_got), np.stack(s_ref), tol, (2, 3))
    unused = sorted(set(range(c["pool"].shape[0])) - set(c["slots"]))
    assert torch.equal(got_pool[unused], c["pool"][unused])


def _exact(d, io):
    """verify + commit runs the same SIMT step as kda_verify for every d and I/O type"""
    return True


@pytest.mark.parametrize("d,io", [(128, "bf16"), (128, "fp32"), (64, "bf16")])
def test_verify_commit_equals_verify_and_snapshot(cuda_device, d, io):
    """The fused step equals kda_verify of the previous batch with per-token states,
    kda_snapshot of the accepted token's state into the slot, then kda_verify of this
    batch: committed states and outputs bit for bit."""
    H, n_seq = 16, 64
    c = _case(801, n_seq, H, d, io, cuda_device)
    pool_a = c["pool"].to(cuda_device)
    pool_b = pool_a.clone()
    # reference path
    dp, dc, cp, cd = c["dp"], c["dc"], c["cp"], c["cd"]
    ts = torch.empty((int(cp[-1]), H, d, d), device=cuda_device)
    op = torch.empty_like(dp["v"])
    K.kda_verify(dp["q"], dp["k"], dp["v"], dp["g"], dp["beta"], cp, c["slots_d"], pool_a, ts, op)
    keep = [s for s in range(n_seq) if c["acc"][s] > 0]
    src = torch.tensor([int(cp[s]) + c["acc"][s] - 1 for s in keep], dtype=torch.int64,
                       device=cuda_device)
    dst = torch.tensor([c["slots"][s] for s in keep], dtype=torch.int64, device=cuda_device)
    K.kda_snapshot(src, dst, ts, pool_a)
    ts2 = torch.empty((int(cd[-1]), H, d, d), device=cuda_device)
    o_ref = torch.empty_like(dc["v"])
    K.kda_verify(dc["q"], dc["k"], dc["v"], dc["g"], dc["beta"], cd, c["slots_d"], pool_a, ts2, o_ref)
    # fused
    o = _fused(c, pool_b)
    assert K.kda_check_device_status() == 0
    ex = _exact(d, io)
    assert same_states(pool_b, pool_a, ex)
    assert same_outputs(o, o_ref, ex)


@pytest.mark.parametrize("io", ["bf16", "fp32"])
def test_verify_commit_writes_block_boundary_snapshots(cuda_device, io):
    """Sequences whose committed tokens cross a multiple of snap_interval write the
    state at that position to their snapshot row (bit-identical to the per-token state
    of kda_verify); the others leave their row untouched."""
    H, d, n_seq, snap = 4, 128, 24, 64
    c = _case(901, n_seq, H, d, io, cuda_device)
    cp = c["cp"]
    # positions a few tokens before a boundary, so that some accepted prefixes cross it
    pos = [snap * (s + 1) - 1 - (s % 6) for s in range(n_seq)]
    rows = list(range(n_seq))
    sn = torch.full((n_seq, H, d, d), float("nan"), device=cuda_device)
    pool_b = c["pool"].to(cuda_device)
    _fused(c, pool_b, pos=torch.tensor(pos, dtype=torch.int64, device=cuda_device),
           snap_interval=snap, snap_row=torch.tensor(rows, dtype=torch.int64, device=cuda_device),
           snapshots=sn)
    assert K.kda_check_device_status() == 0
    dp = c["dp"]
    ts = torch.empty((int(cp[-1]), H, d, d), device=cuda_device)
    op = torch.empty_like(dp["v"])
    K.kda_verify(dp["q"], dp["k"], dp["v"], dp["g"], dp["beta"], cp, c["slots_d"],
                 c["pool"].to(cuda_device), ts, op)
    crossed = 0
    for s in range(n_seq):
        j = snap * (pos[s] // snap + 1) - pos[s] - 1        # token index that lands on it
        if j < c["acc"][s]:
            assert same_states(sn[s], ts[int(cp[s]) + j], _exact(d, io)), s
            crossed += 1
        else:
            assert torch.isnan(sn[s]).all(), s
    assert 0 < crossed < n_seq


def test_verify_commit_drain_and_range(cuda_device):
    """An empty draft batch only commits; an acceptance count above the previous batch
    length is a range error that skips that sequence and no other."""
    H, d, n_seq = 2, 64, 5
    c = _case(990, n_seq, H, d, "bf16", cuda_device)
    pool_d = c["pool"].to(cuda_device)
    empty = {k: v[:0] for k, v in c["dc"].items()}
    cd0 = np.zeros(n_seq + 1, dtype=np.int32)
    o = torch.empty((0, H, d), dtype=torch.bfloat16, device=cuda_device)
    bad = list(c["acc"])
    m1 = int(c["cp"][2] - c["cp"][1])
    bad[1] = m1 + 1
    K.kda_verify_commit(c["dp"], torch.tensor(bad, dtype=torch.int32, device=cuda_device),
                        c["cp"], empty["q"], empty["k"], empty["v"], empty["g"], empty["beta"],
                        cd0, c["slots_d"], pool_d, o)
    assert K.kda_check_device_status() == 7
    got = pool_d.cpu()
    assert torch.equal(got[c["slots"][1]], c["pool"][c["slots"][1]])
    xp = c["xp"]
    for s in (0, 2, 3, 4):
        a, na = int(c["cp"][s]), c["acc"][s]
        slot = c["slots"][s]
        if na == 0:
            assert torch.equal(got[slot], c["pool"][slot])
            continue
        _, st, _ = native.oracle_sequence(xp["q"][a:a + na], xp["k"][a:a + na], xp["v"][a:a + na],
                                          xp["g"][a:a + na], xp["beta"][a:a + na], c["pool"][slot])
        check_states("drained state", got[slot].double().numpy()[None], st[None], TOL_BF16, (2, 3))


@pytest.mark.parametrize("io", ["bf16", "fp32"])
def test_mixed_step_decode_append_and_verify_in_one_launch(cuda_device, io):
    """One launch serving three kinds of sequences (continuous batching): plain decode
    (one token, committed), a short prefill appended to a live sequence (several tokens,
    committed) and speculative sequences (the previous step's accepted prefix committed,
    this step's drafts only verified). Committed states equal kda_decode / kda_verify's
    per-token states and outputs equal kda_verify's bit for bit, and a block-boundary
    snapshot falling among appended tokens is written."""
    H, d, n_seq, snap = 8, 128, 12, 64
    c = _case(1201, n_seq, H, d, io, cuda_device)
    ex = _exact(d, io)
    odt = torch.bfloat16 if io == "bf16" else torch.float32
    cp, cd = c["cp"], c["cd"]
    kind = ["decode", "append", "verify"] * 4
    # decode and append sequences commit nothing of the previous batch
    acc = [a if kind[s] == "verify" else 0 for s, a in enumerate(c["acc"])]
    lens = np.diff(cd).tolist()
    for s in range(n_seq):
        if kind[s] == "decode":
            lens[s] = 1
    cd = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    xc = synth.token_inputs(1202, int(cd[-1]), H, d, d, io=io)
    dc = {k: v.to(cuda_device) for k, v in xc.items()}
    pos = [snap * (s + 1) - 2 for s in range(n_seq)]          # boundaries 2 tokens ahead
    sn = torch.full((n_seq, H, d, d), float("nan"), device=cuda_device)
    pool_b = c["pool"].to(cuda_device)
    o = torch.empty((int(cd[-1]), H, d), dtype=odt, device=cuda_device)
    cnew = torch.tensor([k != "verify" for k in kind], dtype=torch.uint8, device=cuda_device)
    K.kda_verify_commit(c["dp"], torch.tensor(acc, dtype=torch.int32, device=cuda_device), cp,
                        dc["q"], dc["k"], dc["v"], dc["g"], dc["beta"], cd, c["slots_d"], pool_b, o,
                        pos=torch.tensor(pos, dtype=torch.int64, device=cuda_device),
                        snap_interval=snap,
                        snap_row=torch.arange(n_seq, dtype=torch.int64, device=cuda_device),
                        snapshots=sn, commit_new=cnew)
    assert K.kda_check_device_status() == 0
    # reference: commit the verify sequences' accepted prefix, then kda_verify of this batch
    pool_a = c["pool"].to(cuda_device)
    dp = c["dp"]
    ts = torch.empty((int(cp[-1]), H, d, d), device=cuda_device)
    K.kda_verify(dp["q"], dp["k"], dp["v"], dp["g"], dp["beta"], cp, c["slots_d"], pool_a, ts,
                 torch.empty_like(dp["v"]))
    keep = [s for s in range(n_seq) if acc[s] > 0]
    K.kda_snapshot(torch.tensor([int(cp[s]) + acc[s] - 1 for s in keep], dtype=torch.int64,
                                device=cuda_device),
                   torch.tensor([c["slots"][s] for s in keep], dtype=torch.int64, device=cuda_device),
                   ts, pool_a)
    ts2 = torch.empty((int(cd[-1]), H, d, d), device=cuda_device)
    o_ref = torch.empty_like(o)
    K.kda_verify(dc["q"], dc["k"], dc["v"], dc["g"], dc["beta"], cd, c["slots_d"], pool_a, ts2, o_ref)
    assert same_outputs(o, o_ref, ex)
    for s in range(n_seq):
        slot = c["slots"][s]
        if kind[s] == "verify":
            assert same_states(pool_b[slot], pool_a[slot], ex), s
            assert torch.isnan(sn[s]).all() or acc[s] >= 2
        else:
            assert same_states(pool_b[slot], ts2[int(cd[s + 1]) - 1], ex), s   # after the last token
            if lens[s] >= 2:                                                  # boundary at token 1
                assert same_states(sn[s], ts2[int(cd[s]) + 1], ex), s
            else:
                assert torch.isnan(sn[s]).all(), s
    # the decode sequences equal kda_decode itself
    dec = [s for s in range(n_seq) if kind[s] == "decode"]
    rows = torch.tensor([int(cd[s]) for s in dec], device=cuda_device)
    pool_d = c["pool"].to(cuda_device)
    od = torch.empty((len(dec), H, d), dtype=odt, device=cuda_device)
    K.kda_decode(dc["q"][rows].contiguous(), dc["k"][rows].contiguous(), dc["v"][rows].contiguous(),
                 dc["g"][rows].contiguous(), dc["beta"][rows].contiguous(),
                 c["slots_d"][dec].contiguous(), pool_d, od)
    for i, s in enumerate(dec):
        assert same_states(pool_b[c["slots"][s]], pool_d[c["slots"][s]], ex)
        assert same_outputs(o[int(cd[s])], od[i], ex)


def test_verify_commit_empty_items_among_others(cuda_device):
    """Sequences with nothing accepted and no drafts (no work at all), nothing accepted
    only, or no drafts only, interleaved with the rest: the persistent grid's producer
    skips the empty items while it prefetches across item boundaries, and every other
    sequence still equals kda_verify + kda_snapshot + kda_verify bit for bit."""
    H, d, n_seq = 4, 64, 300
    c = _case(1301, n_seq, H, d, "bf16", cuda_device, lo=0, hi=8)
    cp, cd = c["cp"], c["cd"]
    assert (np.diff(cp) == 0).any() and (np.diff(cd) == 0).any()
    pool_a = c["pool"].to(cuda_device)
    pool_b = pool_a.clone()
    dp, dc = c["dp"], c["dc"]
    ts = torch.empty((max(1, int(cp[-1])), H, d, d), device=cuda_device)
    K.kda_verify(dp["q"], dp["k"], dp["v"], dp["g"], dp["beta"], cp, c["slots_d"], pool_a, ts,
                 torch.empty_like(dp["v"]))
    keep = [s for s in range(n_seq) if c["acc"][s] > 0]
    K.kda_snapshot(torch.tensor([int(cp[s]) + c["acc"][s] - 1 for s in keep], dtype=torch.int64,
                                device=cuda_device),
                   torch.tensor([c["slots"][s] for s in keep], dtype=torch.int64, device=cuda_device),
                   ts, pool_a)
    o_ref = torch.empty_like(dc["v"])
    ts2 = torch.empty((max(1, int(cd[-1])), H, d, d), device=cuda_device)
    K.kda_verify(dc["q"], dc["k"], dc["v"], dc["g"], dc["beta"], cd, c["slots_d"], pool_a, ts2, o_ref)
    o = _fused(c, pool_b)
    assert K.kda_check_device_status() == 0
    assert torch.equal(pool_b, pool_a)
    assert torch.equal(o, o_ref)
