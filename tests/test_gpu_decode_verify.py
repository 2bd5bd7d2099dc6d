"""GPU parity of kda_decode, kda_verify and kda_snapshot against the fp64
oracle (token recurrence; Kimi K3 technical FAQ, "What is KDA"), through the C
ABI. Workload shapes: 512 sequences x 64 heads of d_k = d_v = 128 fp32 states
N(0, 0.1^2), bf16 q/k/v, one decode token, then verify drafts of 1..8 tokens.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from hybrid_linear_attention_04_b200 import kda as K
from kda_cases import TOL_BF16, TOL_FP32, blockwise_err, check_outputs, check_states, to_np
from oracle import native

pytestmark = pytest.mark.gpu


def _decode_case(seed, n_seq, H, d, io, dev, n_extra=7):
    n_slots = n_seq + n_extra
    x = synth.token_inputs(seed, n_seq, H, d, d, io=io)
    pool = synth.states(seed, n_slots, H, d, d, std=0.1)
    slots = torch.tensor(synth.permutation(seed, n_slots, "slots")[:n_seq], dtype=torch.int32)
    return x, pool, slots


def _oracle_decode(x, pool, slots):
    n_seq, H, d = x["q"].shape
    o = np.empty((n_seq, H, d))
    S = np.empty((n_seq, H, d, d))
    for s in range(n_seq):
        oo, ss, _ = native.oracle_sequence(x["q"][s:s + 1], x["k"][s:s + 1], x["v"][s:s + 1],
                                           x["g"][s:s + 1], x["beta"][s:s + 1],
                                           pool[int(slots[s])])
        o[s], S[s] = oo[0], ss
    return o, S


@pytest.mark.parametrize("d,io,H,n_seq", [(128, "bf16", 64, 512), (128, "fp32", 4, 9),
                                          (64, "bf16", 3, 17), (32, "fp32", 2, 5)])
def test_decode_matches_oracle(cuda_device, d, io, H, n_seq):
    x, pool, slots = _decode_case(100 + d, n_seq, H, d, io, cuda_device)
    dv = {k: v.to(cuda_device) for k, v in x.items()}
    pool_d = pool.to(cuda_device)
    slots_d = slots.to(cuda_device)
    o = torch.empty_like(dv["v"])
    K.kda_decode(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"], slots_d, pool_d, o)
    assert K.kda_check_device_status() == 0
    o_ref, S_ref = _oracle_decode(x, pool, slots)
    tol = TOL_BF16 if io == "bf16" else TOL_FP32
    check_outputs("o", to_np(o), o_ref, tol, np.arange(n_seq + 1))
    got = to_np(pool_d)
    check_states("state", got[slots.numpy()], S_ref, tol, (2, 3))
    # rows that no sequence uses are untouched, bit for bit
    unused = sorted(set(range(pool.shape[0])) - set(slots.tolist()))
    assert torch.equal(pool_d[unused].cpu(), pool[unused])


def test_decode_bad_slot_sets_range_status(cuda_device):
    x, pool, _ = _decode_case(7, 4, 2, 32, "fp32", cuda_device, n_extra=0)
    dv = {k: v.to(cuda_device) for k, v in x.items()}
    pool_d = pool.to(cuda_device)
    slots = torch.tensor([0, 1, 4, 2], dtype=torch.int32, device=cuda_device)   # 4 is out of range
    o = torch.zeros_like(dv["v"])
    K.kda_decode(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"], slots, pool_d, o)
    assert K.kda_check_device_status() == 7
    assert K.kda_check_device_status() == 0          # the check clears the word
    assert torch.equal(pool_d[3].cpu(), pool[3])


def _verify_case(seed, n_seq, H, d, io, lo=1, hi=8):
    lens = synth.draft_lengths(seed, n_seq, lo, hi)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = synth.token_inputs(seed, int(cu[-1]), H, d, d, io=io)
    pool = synth.states(seed, n_seq + 3, H, d, d, std=0.1)
    slots = torch.tensor(synth.permutation(seed, n_seq + 3, "slots")[:n_seq], dtype=torch.int32)
    return x, cu, pool, slots


@pytest.mark.parametrize("d,io,H,n_seq", [(128, "bf16", 64, 512), (128, "fp32", 2, 6),
                                          (64, "bf16", 4, 11)])
def test_verify_matches_oracle_and_rollback(cuda_device, d, io, H, n_seq):
    x, cu, pool, slots = _verify_case(200 + d, n_seq, H, d, io)
    dv = {k: v.to(cuda_device) for k, v in x.items()}
    pool_d = pool.to(cuda_device)
    slots_d = slots.to(cuda_device)
    T = int(cu[-1])
    ts = torch.empty((T, H, d, d), dtype=torch.float32, device=cuda_device)
    o = torch.empty_like(dv["v"])
    K.kda_verify(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"], cu, slots_d, pool_d, ts, o)
    assert K.kda_check_device_status() == 0
    assert torch.equal(pool_d.cpu(), pool)           # the source pool is only read
    tol = TOL_BF16 if io == "bf16" else TOL_FP32
    o_got, ts_got = to_np(o), ts.cpu().numpy()
    o_all, ts_all = np.zeros_like(o_got), np.zeros(ts_got.shape)
    for s in range(n_seq):
        a, b = int(cu[s]), int(cu[s + 1])
        oo, _, sn = native.oracle_sequence(x["q"][a:b], x["k"][a:b], x["v"][a:b], x["g"][a:b],
                                           x["beta"][a:b], pool[int(slots[s])], None, 0, 1)
        assert blockwise_err(o_got[a:b], oo, (2,)) <= tol, s
        assert blockwise_err(ts_got[a:b], sn, (2, 3)) <= tol, s
        o_all[a:b], ts_all[a:b] = oo, sn
    check_outputs("o", o_got, o_all, tol, cu)
    check_states("token states", ts_got, ts_all, tol, (2, 3))
    # rollback: commit the state of a seeded accepted prefix into the live slot
    acc = synth.randint(200 + d, "misc", n_seq, 0, 8)
    src = [int(cu[s]) + min(acc[s], int(cu[s + 1] - cu[s])) - 1 for s in range(n_seq)]
    keep = [s for s in range(n_seq) if src[s] >= int(cu[s])]
    src_i = torch.tensor([src[s] for s in keep], dtype=torch.int64, device=cuda_device)
    dst_i = torch.tensor([int(slots[s]) for s in keep], dtype=torch.int64, device=cuda_device)
    K.kda_snapshot(src_i, dst_i, ts, pool_d)
    assert K.kda_check_device_status() == 0
    for j, s in enumerate(keep):
        assert torch.equal(pool_d[int(slots[s])], ts[src[s]])


def test_verify_states_equal_repeated_decode_bitwise(cuda_device):
    """Verify's state after token j is bit-identical to j kda_decode calls
    (the two kernels share the per-token step)."""
    H, d, n_seq = 8, 128, 16
    x, cu, pool, slots = _verify_case(300, n_seq, H, d, "bf16")
    dv = {k: v.to(cuda_device) for k, v in x.items()}
    pool_d = pool.to(cuda_device)
    slots_d = slots.to(cuda_device)
    T = int(cu[-1])
    ts = torch.empty((T, H, d, d), dtype=torch.float32, device=cuda_device)
    o = torch.empty_like(dv["v"])
    K.kda_verify(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"], cu, slots_d, pool_d, ts, o)
    lens = np.diff(cu)
    live = pool_d.clone()
    o1 = torch.empty((n_seq, H, d), dtype=dv["v"].dtype, device=cuda_device)
    for j in range(int(lens.max())):
        act = [s for s in range(n_seq) if lens[s] > j]
        rows = torch.tensor([int(cu[s]) + j for s in act], device=cuda_device)
        sl = slots_d[act].contiguous()
        oo = o1[:len(act)]
        K.kda_decode(dv["q"][rows].contiguous(), dv["k"][rows].contiguous(),
                     dv["v"][rows].contiguous(), dv["g"][rows].contiguous(),
                     dv["beta"][rows].contiguous(), sl, live, oo)
        for i, s in enumerate(act):
            assert torch.equal(live[int(slots[s])], ts[int(cu[s]) + j])
            assert torch.equal(oo[i], o[int(cu[s]) + j])
    assert K.kda_check_device_status() == 0


def test_snapshot_copies_bit_exact_and_checks_range(cuda_device):
    H, d = 4, 64
    src = synth.states(5, 10, H, d, d, std=1.0).to(cuda_device)
    dst = torch.full((6, H, d, d), float("nan"), device=cuda_device)
    si = torch.tensor([3, 0, 9], dtype=torch.int64, device=cuda_device)
    di = torch.tensor([5, 1, 0], dtype=torch.int64, device=cuda_device)
    K.kda_snapshot(si, di, src, dst)
    assert K.kda_check_device_status() == 0
    for a, b in zip(si.tolist(), di.tolist()):
        assert torch.equal(dst[b], src[a])
    assert torch.isnan(dst[[2, 3, 4]]).all()
    bad = torch.tensor([10], dtype=torch.int64, device=cuda_device)
    K.kda_snapshot(bad, di[:1], src, dst)
    assert K.kda_check_device_status() == 7


def test_verify_more_sequences_than_one_launch(cuda_device):
    """1030 sequences: the library splits the batch into launches of at most
    KDA_SEQS_PER_LAUNCH sequences; outputs and per-token states match the oracle."""
    H, d, n_seq = 2, 64, 1030
    x, cu, pool, slots = _verify_case(500, n_seq, H, d, "bf16", lo=1, hi=3)
    dv = {k: v.to(cuda_device) for k, v in x.items()}
    pool_d = pool.to(cuda_device)
    T = int(cu[-1])
    ts = torch.empty((T, H, d, d), dtype=torch.float32, device=cuda_device)
    o = torch.empty_like(dv["v"])
    K.kda_verify(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"], cu, slots.to(cuda_device), pool_d,
                 ts, o)
    assert K.kda_check_device_status() == 0
    o_got, ts_got = to_np(o), ts.cpu().numpy()
    for s in range(0, n_seq, 7):
        a, b = int(cu[s]), int(cu[s + 1])
        oo, _, sn = native.oracle_sequence(x["q"][a:b], x["k"][a:b], x["v"][a:b], x["g"][a:b],
                                           x["beta"][a:b], pool[int(slots[s])], None, 0, 1)
        assert blockwise_err(o_got[a:b], oo, (2,)) <= TOL_BF16, s
        assert blockwise_err(ts_got[a:b], sn, (2, 3)) <= TOL_BF16, s
