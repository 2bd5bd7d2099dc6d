"""GPU parity on the degenerate inputs of the gated delta rule (Kimi K3 technical
FAQ, "What is KDA, and why does a serving engineer care?"), through the C ABI,
against the fp64 oracle on the same inputs:

- no write (beta = 0): the state only decays;
- no forgetting (g = 0, alpha = 1);
- zero keys: nothing is erased or written, the outputs read the decayed state;
- zero queries: every output is exactly zero;
- full-strength writes of basis keys without decay (beta = 1, g = 0): each token
  replaces its key's row of the state by v;
- calls without tokens: the states pass through bit for bit.

Every prefill path (tensor cores in two launches or one, CUDA cores), decode and
verify run each case.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from hybrid_linear_attention_04_b200 import kda as K
from kda_cases import TOL_BF16, check_outputs, check_states, oracle_prefill, to_np
from oracle import native
from test_gpu_prefill import check, path, run_prefill  # noqa: F401  (path is a fixture)

pytestmark = pytest.mark.gpu

CASES = ["no_write", "no_forgetting", "zero_keys", "zero_queries", "basis_overwrite"]


def _degenerate(x: dict, case: str) -> dict:
    """The seeded inputs with one degenerate feature imposed (CPU tensors, in place)."""
    T, H, d = x["k"].shape
    if case == "no_write":
        x["beta"].zero_()
    elif case == "no_forgetting":
        x["g"].zero_()
    elif case == "zero_keys":
        x["k"].zero_()
    elif case == "zero_queries":
        x["q"].zero_()
    elif case == "basis_overwrite":
        x["g"].zero_()
        x["beta"].fill_(1.0)
        x["k"].zero_()
        idx = (np.arange(T)[:, None] * 5 + 3 * np.arange(H)[None, :]) % d
        for t in range(T):
            for h in range(H):
                x["k"][t, h, int(idx[t, h])] = 1.0
    else:
        raise ValueError(case)
    return x


def _inputs(seed, T, H, d, io, case, device):
    x = _degenerate(synth.token_inputs(seed, T, H, d, d, io=io), case)
    return x, {k: v.to(device) for k, v in x.items()}


@pytest.mark.parametrize("case", CASES)
def test_prefill_degenerate_inputs(cuda_device, path, case):
    lens = [1, 63, 64, 65, 200]
    H, d, C = 3, 128, 64
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x, dev = _inputs(700 + CASES.index(case), int(cu[-1]), H, d, "bf16", case, cuda_device)
    start = [0, 64, 0, 128, 64]
    s0 = synth.states(701, len(lens), H, d, d, std=0.1)
    o, sout, snaps, offs = run_prefill(dev, cu, H, d, C, "bf16", start, s0.to(cuda_device), C,
                                       cuda_device)
    check(o, sout, snaps, offs, oracle_prefill(x, cu, start, s0, C), "bf16", cu)
    if case == "zero_queries":
        assert bool((o == 0).all())


def test_prefill_without_tokens_passes_states_through(cuda_device, path):
    H, d = 2, 128
    cu = np.zeros(3, dtype=np.int32)
    empty = {"q": torch.empty((0, H, d), dtype=torch.bfloat16, device=cuda_device),
             "k": torch.empty((0, H, d), dtype=torch.bfloat16, device=cuda_device),
             "v": torch.empty((0, H, d), dtype=torch.bfloat16, device=cuda_device),
             "g": torch.empty((0, H, d), device=cuda_device),
             "beta": torch.empty((0, H), device=cuda_device)}
    s0 = synth.states(702, 2, H, d, d, std=0.1).to(cuda_device)
    o, sout, snaps, offs = run_prefill(empty, cu, H, d, 64, "bf16", None, s0, 0, cuda_device)
    assert o.numel() == 0 and int(offs[-1]) == 0
    assert torch.equal(sout, s0)


def _pool_case(seed, n_seq, H, d):
    pool = synth.states(seed, n_seq + 2, H, d, d, std=0.1)
    slots = torch.tensor(synth.permutation(seed, n_seq + 2, "slots")[:n_seq], dtype=torch.int32)
    return pool, slots


@pytest.mark.parametrize("case", CASES)
def test_decode_degenerate_inputs(cuda_device, case):
    H, d, n_seq = 4, 128, 9
    x, dev = _inputs(720 + CASES.index(case), n_seq, H, d, "bf16", case, cuda_device)
    pool, slots = _pool_case(721, n_seq, H, d)
    pool_d, slots_d = pool.to(cuda_device), slots.to(cuda_device)
    o = torch.empty_like(dev["v"])
    K.kda_decode(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], slots_d, pool_d, o)
    assert K.kda_check_device_status() == 0
    o_ref, S_ref = np.empty((n_seq, H, d)), np.empty((n_seq, H, d, d))
    for s in range(n_seq):
        oo, ss, _ = native.oracle_sequence(x["q"][s:s + 1], x["k"][s:s + 1], x["v"][s:s + 1],
                                           x["g"][s:s + 1], x["beta"][s:s + 1],
                                           pool[int(slots[s])])
        o_ref[s], S_ref[s] = oo[0], ss
    check_outputs("o", to_np(o), o_ref, TOL_BF16, np.arange(n_seq + 1))
    check_states("state", to_np(pool_d)[slots.numpy()], S_ref, TOL_BF16, (2, 3))
    if case == "zero_queries":
        assert bool((o == 0).all())


@pytest.mark.parametrize("case", CASES)
def test_verify_degenerate_inputs(cuda_device, case):
    H, d, n_seq = 4, 128, 7
    lens = synth.draft_lengths(740, n_seq, 1, 8)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    x, dev = _inputs(740 + CASES.index(case), T, H, d, "bf16", case, cuda_device)
    pool, slots = _pool_case(741, n_seq, H, d)
    pool_d, slots_d = pool.to(cuda_device), slots.to(cuda_device)
    ts = torch.empty((T, H, d, d), dtype=torch.float32, device=cuda_device)
    o = torch.empty_like(dev["v"])
    K.kda_verify(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], cu, slots_d, pool_d, ts, o)
    assert K.kda_check_device_status() == 0
    o_ref, ts_ref = np.empty((T, H, d)), np.empty((T, H, d, d))
    for s in range(n_seq):
        a, b = int(cu[s]), int(cu[s + 1])
        oo, _, sn = native.oracle_sequence(x["q"][a:b], x["k"][a:b], x["v"][a:b], x["g"][a:b],
                                           x["beta"][a:b], pool[int(slots[s])], None, 0, 1)
        o_ref[a:b], ts_ref[a:b] = oo, sn
    check_outputs("o", to_np(o), o_ref, TOL_BF16, cu)
    check_states("token states", ts.cpu().numpy(), ts_ref, TOL_BF16, (2, 3))
    if case == "zero_queries":
        assert bool((o == 0).all())


def test_decode_and_verify_without_sequences(cuda_device):
    """Zero sequences: nothing is launched and nothing changes."""
    H, d = 2, 128
    pool, _ = _pool_case(760, 1, H, d)
    pool_d = pool.to(cuda_device)
    e3 = torch.empty((0, H, d), dtype=torch.bfloat16, device=cuda_device)
    eg = torch.empty((0, H, d), device=cuda_device)
    eb = torch.empty((0, H), device=cuda_device)
    es = torch.empty((0,), dtype=torch.int32, device=cuda_device)
    n0 = K.kda_launch_count()
    K.kda_decode(e3, e3, e3, eg, eb, es, pool_d, e3.clone())
    ts = torch.empty((0, H, d, d), device=cuda_device)
    K.kda_verify(e3, e3, e3, eg, eb, np.zeros(1, dtype=np.int32), es, pool_d, ts, e3.clone())
    assert K.kda_check_device_status() == 0
    assert K.kda_launch_count() == n0
    assert torch.equal(pool_d.cpu(), pool)
