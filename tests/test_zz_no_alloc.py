"""kda_prefill_noalloc: the prefill call that neither allocates nor takes a caller
workspace. It runs the two-launch prefill on the library's fixed device scratch:
in one piece when the call's workspace fits there, else as pieces (groups of whole
sequences, and windows of whole chunks of a sequence too long for the scratch). Both
are checked against the fp64 oracle (token recurrence; Kimi K3 technical FAQ, "What is
KDA") and bit for bit against kda_prefill with a caller workspace.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import synth
from hybrid_linear_attention_04_b200 import build as kbuild
from hybrid_linear_attention_04_b200 import kda as K
from kda_cases import (blockwise_err, check_outputs, check_states, oracle_prefill, packed_inputs,
                       to_np, tol_for)

PACKET = 75776      # workspace bytes per (64-token chunk row, head)


@pytest.fixture(scope="module", autouse=True)
def built():
    kbuild.build()


def test_capacity_and_validation_on_host():
    """Host-only: the scratch is 64 MiB, and arguments are checked before any CUDA call."""
    L = K.lib()
    assert K.kda_prefill_noalloc_capacity() == 64 << 20
    A = ctypes.c_void_p(0x10000)
    cu = np.array([0, 64], dtype=np.int32)

    def call(dims, cu, n_seq=None):
        return L.kda_prefill_noalloc(ctypes.byref(dims), len(cu) - 1 if n_seq is None else n_seq,
                                     cu.ctypes.data_as(ctypes.c_void_p), None, A, A, A, A, A, None,
                                     A, A, 0, None, None)

    assert call(K.kda_dims(4, 96, 96, 64, 0, 0.0), cu) == 2          # unsupported head dim
    assert call(K.kda_dims(4, 128, 128, 64, 0, 0.0), np.array([0, 64, 10], np.int32)) == 1
    assert call(K.kda_dims(4, 128, 128, 64, 0, 0.0), np.array([0], np.int32), n_seq=0) == 0


def _run(fn, x, dev, cu, H, d, start, s0, snap, **kw):
    T, n = int(cu[-1]), len(cu) - 1
    o = torch.empty((T, H, d), dtype=dev["v"].dtype, device=dev["v"].device)
    so = torch.empty((n, H, d, d), device=o.device)
    offs, _ = K.kda_snapshot_plan(cu, start, snap)
    sn = torch.full((int(offs[-1]) + 1, H, d, d), float("nan"), device=o.device)
    fn(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], cu, o, state_out=so,
       state_in=None if s0 is None else s0.to(o.device), start_pos=start, snap_interval=snap,
       snapshots=sn, chunk=64, **kw)
    assert K.kda_check_device_status() == 0
    assert torch.isnan(sn[int(offs[-1])]).all()
    return o, so, sn[:int(offs[-1])]


@pytest.mark.gpu
def test_fits_in_scratch_two_launches_and_matches(cuda_device):
    """A ragged batch whose workspace fits the scratch: two launches (prep, chain), the
    oracle's results, and the same bits as kda_prefill with a caller workspace."""
    lens, H, d = [70, 0, 256, 129], 2, 128
    x, dev, cu = packed_inputs(61, lens, H, d, "bf16", cuda_device)
    assert K.kda_prefill_workspace_size(dev["q"], dev["v"], cu) <= K.kda_prefill_noalloc_capacity()
    start = [0, 64, 128, 0]
    s0 = synth.states(62, len(lens), H, d, d, std=0.1)
    n0 = K.kda_launch_count()
    got = _run(K.kda_prefill_noalloc, x, dev, cu, H, d, start, s0, 128)
    assert K.kda_launch_count() - n0 == 2
    ref = oracle_prefill(x, cu, start, s0, 128)
    tol = tol_for("bf16")
    check_outputs("o", to_np(got[0]), ref[0], tol, cu)
    check_states("state", to_np(got[1]), ref[1], tol, (2, 3))
    check_states("snapshots", got[2].cpu().numpy(), ref[2], tol, (2, 3))
    ws = torch.empty(K.kda_prefill_workspace_size(dev["q"], dev["v"], cu), dtype=torch.uint8,
                     device=cuda_device)
    again = _run(K.kda_prefill, x, dev, cu, H, d, start, s0, 128, workspace=ws)
    for a, b in zip(got, again):
        assert torch.equal(a, b)


@pytest.mark.gpu
def test_larger_than_scratch_runs_in_windows(cuda_device):
    """1024 tokens x 64 heads need (16 + 1) x 64 packets (82 MB) > 64 MiB: two windows
    of the two-launch path (704 + 320 tokens, the state handed over in fp32 between them),
    the oracle's results, and the same bits as kda_prefill with a full workspace."""
    T, H, d = 1024, 64, 128
    x, dev, cu = packed_inputs(63, [T], H, d, "bf16", cuda_device)
    need = K.kda_prefill_workspace_size(dev["q"], dev["v"], cu)
    assert need == (T // 64 + 1) * H * PACKET > K.kda_prefill_noalloc_capacity()
    s0 = synth.states(64, 1, H, d, d, std=0.1)
    n0 = K.kda_launch_count()
    got = _run(K.kda_prefill_noalloc, x, dev, cu, H, d, [128], s0, 256)
    assert K.kda_launch_count() - n0 == 4
    ref = oracle_prefill(x, cu, [128], s0, 256)
    tol = tol_for("bf16")
    # outputs per (token, head) row as well as per head: the first tokens' rows scale
    # with q.k, and only an fp32-accurate decayed QK^T keeps them within the tolerance
    # where that product nearly cancels
    check_outputs("o", to_np(got[0]), ref[0], tol, cu)
    check_states("state", to_np(got[1]), ref[1], tol, (2, 3))
    check_states("snapshots", got[2].cpu().numpy(), ref[2], tol, (2, 3))
    ws = torch.empty(need, dtype=torch.uint8, device=cuda_device)
    again = _run(K.kda_prefill, x, dev, cu, H, d, [128], s0, 256, workspace=ws)
    for a, b in zip(got, again):
        assert torch.equal(a, b)


@pytest.mark.gpu
def test_ragged_batch_larger_than_scratch_in_pieces(cuda_device):
    """A ragged 64-head batch whose packets exceed the scratch: short sequences grouped,
    a long one in windows, zero-length and resumed sequences among them; the same bits as
    kda_prefill with a full workspace (outputs, final states, snapshots)."""
    lens, H, d = [130, 0, 1500, 64, 700, 1], 64, 128
    x, dev, cu = packed_inputs(65, lens, H, d, "bf16", cuda_device)
    need = K.kda_prefill_workspace_size(dev["q"], dev["v"], cu)
    assert need > K.kda_prefill_noalloc_capacity()
    start = [0, 64, 256, 0, 512, 0]
    s0 = synth.states(66, len(lens), H, d, d, std=0.1)
    got = _run(K.kda_prefill_noalloc, x, dev, cu, H, d, start, s0, 128)
    ws = torch.empty(need, dtype=torch.uint8, device=cuda_device)
    again = _run(K.kda_prefill, x, dev, cu, H, d, start, s0, 128, workspace=ws)
    for a, b in zip(got, again):
        assert torch.equal(a, b)
