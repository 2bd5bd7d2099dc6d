"""GPU parity of kda_prefill against the fp64 oracle (token recurrence), through
the C ABI: packed ragged batches, initial states, start positions and
block-boundary snapshots (vLLM day-0 blog, "Kimi Delta Attention"), on all three
prefill paths (tensor cores in two launches or one, CUDA cores) where the dims
allow.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from hybrid_linear_attention_04_b200 import kda as K
from kda_cases import (blockwise_err, check_outputs, check_states, oracle_prefill, packed_inputs,
                       to_np, tol_for)

pytestmark = pytest.mark.gpu


# prefill paths: "split" (tensor cores, two launches through a workspace), "fused"
# (tensor cores, one launch, no workspace), "simt" (CUDA cores); dimensions the
# tensor-core kernels do not cover run on the CUDA cores under every setting.
_WS = {"split": "auto", "fused": None, "simt": "auto"}
_mode = {"ws": "auto"}


@pytest.fixture(params=["split", "fused", "simt"])
def path(request):
    K.lib().kda_internal_force_prefill_path(1 if request.param == "simt" else 0)
    _mode["ws"] = _WS[request.param]
    yield request.param
    _mode["ws"] = "auto"
    K.lib().kda_internal_force_prefill_path(0)


def run_prefill(dev, cu, H, d, chunk, io, start=None, s0=None, snap=0, device=None):
    n_seq = len(cu) - 1
    T = int(cu[-1])
    o = torch.empty((T, H, d), dtype=dev["v"].dtype, device=device)
    sout = torch.empty((n_seq, H, d, d), dtype=torch.float32, device=device)
    offs, pos = K.kda_snapshot_plan(cu, start, snap)
    n_snap = int(offs[-1])
    # sentinel-filled snapshot pool with one spare row: only planned rows change
    snaps = torch.full((n_snap + 1, H, d, d), float("nan"), device=device)
    K.kda_prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], cu, o, state_out=sout,
                  state_in=s0, start_pos=start, snap_interval=snap, snapshots=snaps, chunk=chunk,
                  workspace=_mode["ws"])
    assert K.kda_check_device_status() == 0
    return o, sout, snaps, offs


def check(o, sout, snaps, offs, ref, io, cu=None):
    tol = tol_for(io)
    o_ref, s_ref, sn_ref = ref
    check_outputs("o", to_np(o), o_ref, tol, cu)
    check_states("state", to_np(sout), s_ref, tol, (2, 3))
    n_snap = int(offs[-1])
    got = snaps.cpu().numpy()
    assert sn_ref.shape[0] == n_snap
    assert torch.isnan(snaps[n_snap]).all()                      # spare row untouched
    if n_snap:
        assert not np.isnan(got[:n_snap]).any()
        check_states("snapshots", got[:n_snap], sn_ref, tol, (2, 3))


def test_tiny_fp32_workload(cuda_device, path):
    """B=1, H=2, T=64, d=32, chunk 16, fp32 throughout, zero initial state."""
    x, dev, cu = packed_inputs(1000, [64], 2, 32, "fp32", cuda_device)
    o, sout, snaps, offs = run_prefill(dev, cu, 2, 32, 16, "fp32", device=cuda_device)
    check(o, sout, snaps, offs, oracle_prefill(x, cu), "fp32")


@pytest.mark.parametrize("d,chunk,io", [(128, 64, "bf16"), (128, 64, "fp32"), (64, 32, "bf16"),
                                        (32, 16, "fp32"), (128, 16, "bf16")])
def test_ragged_with_state_and_snapshots(cuda_device, path, d, chunk, io):
    lens = [1, chunk - 1, chunk, chunk + 1, 5 * chunk + 7, 0, 8 * chunk]
    H = 3
    x, dev, cu = packed_inputs(400 + d + chunk, lens, H, d, io, cuda_device)
    start = [0, chunk, 0, 3 * chunk, 2 * chunk, chunk, 4 * chunk]
    s0 = synth.states(401, len(lens), H, d, d, std=0.1)
    snap = 2 * chunk
    o, sout, snaps, offs = run_prefill(dev, cu, H, d, chunk, io, start, s0.to(cuda_device), snap,
                                       cuda_device)
    check(o, sout, snaps, offs, oracle_prefill(x, cu, start, s0, snap), io, cu)


def test_snapshot_after_every_chunk(cuda_device, path):
    """snap_interval == chunk: a snapshot is due at every chunk boundary, the case in
    which the two-launch chain writes part of each snapshot directly rather than
    through its staging tile."""
    lens = [200, 64, 130, 1]
    H, d, C = 2, 128, 64
    x, dev, cu = packed_inputs(91, lens, H, d, "bf16", cuda_device)
    start = [0, 64, 128, 192]
    s0 = synth.states(92, len(lens), H, d, d, std=0.1)
    o, sout, snaps, offs = run_prefill(dev, cu, H, d, C, "bf16", start, s0.to(cuda_device), C,
                                       cuda_device)
    assert int(offs[-1]) == 3 + 1 + 2 + 0
    check(o, sout, snaps, offs, oracle_prefill(x, cu, start, s0, C), "bf16", cu)


def test_zero_length_sequence_passes_state_through(cuda_device, path):
    H, d = 2, 128
    x, dev, cu = packed_inputs(9, [0, 70, 0], H, d, "bf16", cuda_device)
    s0 = synth.states(9, 3, H, d, d, std=0.1).to(cuda_device)
    o, sout, snaps, offs = run_prefill(dev, cu, H, d, 64, "bf16", None, s0, 0, cuda_device)
    assert torch.equal(sout[0], s0[0]) and torch.equal(sout[2], s0[2])


def test_prefill_is_deterministic(cuda_device, path):
    H, d = 4, 128
    lens = [300, 129, 64]
    x, dev, cu = packed_inputs(11, lens, H, d, "bf16", cuda_device)
    a = run_prefill(dev, cu, H, d, 64, "bf16", None, None, 64, cuda_device)
    b = run_prefill(dev, cu, H, d, 64, "bf16", None, None, 64, cuda_device)
    for u, v in zip(a[:3], b[:3]):
        assert torch.equal(torch.nan_to_num(u), torch.nan_to_num(v))


def test_resume_from_gpu_snapshot_equals_full_run(cuda_device, path):
    """Prefix caching: resuming from the GPU's own block-boundary snapshot gives
    the same outputs and final state as the uninterrupted GPU run, bit for bit
    (same chunk grid, deterministic kernels)."""
    H, d, C = 4, 128, 64
    T = 1000
    x, dev, cu = packed_inputs(12, [T], H, d, "bf16", cuda_device)
    o, sout, snaps, offs = run_prefill(dev, cu, H, d, C, "bf16", None, None, 256, cuda_device)
    for m in range(int(offs[-1])):
        p = 256 * (m + 1)
        sub = {k: v[p:].contiguous() for k, v in dev.items()}
        cu2 = np.array([0, T - p], dtype=np.int32)
        o2, s2, sn2, offs2 = run_prefill(sub, cu2, H, d, C, "bf16", [p], snaps[m:m + 1].clone(),
                                         256, cuda_device)
        assert torch.equal(o2, o[p:])
        assert torch.equal(s2, sout)
        assert torch.equal(sn2[:int(offs2[-1])], snaps[m + 1:int(offs[-1])])


def test_segment_handoff_equals_one_shot(cuda_device, path):
    """A long sequence processed in segments, each call taking the previous
    call's final state and start position, equals one call, bit for bit."""
    H, d, C, seg = 2, 128, 64, 512
    T = 4 * seg
    x, dev, cu = packed_inputs(13, [T], H, d, "bf16", cuda_device)
    o, sout, snaps, offs = run_prefill(dev, cu, H, d, C, "bf16", None, None, 256, cuda_device)
    state = None
    outs, sn_all = [], []
    for i in range(4):
        sub = {k: v[i * seg:(i + 1) * seg].contiguous() for k, v in dev.items()}
        o2, s2, sn2, offs2 = run_prefill(sub, np.array([0, seg], dtype=np.int32), H, d, C, "bf16",
                                         [i * seg], state, 256, cuda_device)
        outs.append(o2)
        sn_all.append(sn2[:int(offs2[-1])])
        state = s2
    assert torch.equal(torch.cat(outs), o)
    assert torch.equal(state, sout)
    assert torch.equal(torch.cat(sn_all), snaps[:int(offs[-1])])


def test_more_sequences_than_one_launch(cuda_device, path):
    """1030 sequences (more than KDA_SEQS_PER_LAUNCH) split into several launches,
    including zero-length ones, with snapshots and initial states."""
    n_seq, H, d = 1030, 2, 128
    lens = synth.randint(31, "lens", n_seq, 0, 140)
    x, dev, cu = packed_inputs(31, lens, H, d, "bf16", cuda_device)
    start = [64 * m for m in synth.randint(31, "resume", n_seq, 0, 3)]
    s0 = synth.states(31, n_seq, H, d, d, std=0.1)
    o, sout, snaps, offs = run_prefill(dev, cu, H, d, 64, "bf16", start, s0.to(cuda_device), 128,
                                       cuda_device)
    check(o, sout, snaps, offs, oracle_prefill(x, cu, start, s0, 128), "bf16", cu)


@pytest.mark.parametrize("path", ["split", "fused", "simt"])
def test_gates_beyond_one_reference_point_match_oracle(cuda_device, path):
    """Channels whose decay within a chunk exceeds what one reference point per chunk can
    scale (here 3 and 2.5 nats per token: ~190 and ~160 nats per chunk) take the bounded
    references on the tensor-core paths, with their part of the decayed QK^T and KK^T
    from pairwise exponentials: the same results as the oracle, and no status."""
    H, d = 2, 128
    lens = [64, 200, 37]
    x = synth.token_inputs(41, sum(lens), H, d, d, io="bf16")
    x["g"][:, 0, 5] = -3.0                       # one channel of head 0
    x["g"][:, 1, 7:10] = -2.5                    # three channels of head 1
    x["g"][100:140, 1, 40] = -6.0                # a burst in one channel
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    dev = {k: v.to(cuda_device) for k, v in x.items()}
    s0 = synth.states(42, len(lens), H, d, d, std=0.1)
    K.lib().kda_internal_force_prefill_path(1 if path == "simt" else 0)
    try:
        o = torch.empty_like(dev["v"])
        sout = torch.empty((len(lens), H, d, d), device=cuda_device)
        offs, _ = K.kda_snapshot_plan(cu, [0, 64, 128], 64)
        snaps = torch.full((int(offs[-1]) + 1, H, d, d), float("nan"), device=cuda_device)
        K.kda_prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], cu, o, state_out=sout,
                      state_in=s0.to(cuda_device), start_pos=[0, 64, 128], snap_interval=64,
                      snapshots=snaps, chunk=64, workspace=_WS[path])
        assert K.kda_check_device_status() == 0
    finally:
        K.lib().kda_internal_force_prefill_path(0)
    check(o, sout, snaps, offs, oracle_prefill(x, cu, [0, 64, 128], s0, 64), "bf16", cu)


@pytest.mark.parametrize("ws", ["auto", None])
def test_gates_beyond_the_fallback_capacity_are_reported(cuda_device, ws):
    """More channels beyond the single-reference range in one chunk than the tensor-core
    kernels stage (8 in the two-launch path, 4 in the single launch) is reported as
    KDA_ERR_RANGE; the CUDA-core path has no such limit and matches the oracle."""
    H, d, T = 2, 128, 64
    x = synth.token_inputs(43, T, H, d, d, io="bf16")
    x["g"][:, 0, 0:12] = -3.0                    # twelve channels of head 0
    dev = {k: v.to(cuda_device) for k, v in x.items()}
    cu = np.array([0, T], dtype=np.int32)
    o = torch.empty_like(dev["v"])
    K.lib().kda_internal_force_prefill_path(0)
    K.kda_prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], cu, o, chunk=64, workspace=ws)
    assert K.kda_check_device_status() == 7
    K.lib().kda_internal_force_prefill_path(1)
    try:
        sout = torch.empty((1, H, d, d), device=cuda_device)
        K.kda_prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], cu, o, state_out=sout,
                      chunk=64)
        assert K.kda_check_device_status() == 0
    finally:
        K.lib().kda_internal_force_prefill_path(0)
    o_ref, s_ref, _ = oracle_prefill(x, cu)
    check_outputs("o", to_np(o), o_ref, tol_for("bf16"), cu)
    check_states("state", to_np(sout), s_ref, tol_for("bf16"), (2, 3))
