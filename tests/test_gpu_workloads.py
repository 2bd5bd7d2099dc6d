"""Full-size parity of the prefill workloads, in the launch configuration the
benchmark times, against the fp64 oracle (token recurrence; Kimi K3 technical
FAQ, "What is KDA"; snapshots: vLLM day-0 blog, "Kimi Delta Attention").

  prefill 8192 x 64:    every head, outputs, final state and all 32 snapshots.
  ragged 32 sequences:  lognormal lengths (mu = ln 4096, sigma = 1, clipped to
                        [512, 65536]) packed by cu_seqlens; half resume from the
                        GPU's own block-boundary snapshot of a shared 16384-token
                        prefix. The GPU runs every head; the oracle checks four
                        heads, running prefix + sequence itself (resume = full run).
  1M tokens:            16 calls of 65536 tokens handing the state across, with
                        snapshots every 4096 tokens; the oracle checks two heads
                        over the whole length.
Tolerance: 2e-2 for bf16 q/k/v/o with fp32 state, normwise per sequence and
head and, for outputs, per (token, head) row (measures in kda_cases). Snapshot rows
are checked exactly for placement.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from hybrid_linear_attention_04_b200 import kda as K
from kda_cases import TOL_BF16, check_outputs, check_states, to_np
from oracle import native

pytestmark = pytest.mark.gpu

H, D, C = 64, 128, 64


def _prefill(dev_in, cu, start=None, s0=None, snap=0, device=None, workspace="auto"):
    n_seq = len(cu) - 1
    T = int(cu[-1])
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device=device)
    sout = torch.empty((n_seq, H, D, D), device=device)
    offs, pos = K.kda_snapshot_plan(cu, start, snap)
    snaps = torch.full((int(offs[-1]) + 1, H, D, D), float("nan"), device=device)
    K.kda_prefill(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["g"], dev_in["beta"], cu, o,
                  state_out=sout, state_in=s0, start_pos=start, snap_interval=snap, snapshots=snaps,
                  chunk=C, workspace=workspace)
    assert K.kda_check_device_status() == 0
    assert torch.isnan(snaps[-1]).all()
    assert not torch.isnan(snaps[:-1]).any()
    return o, sout, snaps[:-1], offs, pos


_ORACLE_8K = {}


@pytest.mark.parametrize("workspace", ["auto", None], ids=["split", "fused"])
def test_prefill_8k_all_heads(cuda_device, workspace):
    T, snap = 8192, 256
    x = synth.token_inputs(1001, T, H, D, D, io="bf16")
    dev = {k: v.to(cuda_device) for k, v in x.items()}
    cu = np.array([0, T], dtype=np.int32)
    o, sout, snaps, offs, pos = _prefill(dev, cu, snap=snap, device=cuda_device, workspace=workspace)
    assert pos.tolist() == list(range(256, 8193, 256))
    if not _ORACLE_8K:
        _ORACLE_8K["ref"] = native.oracle_sequence(x["q"], x["k"], x["v"], x["g"], x["beta"],
                                                   None, None, 0, snap, out_dtype=np.float32)
    o_ref, s_ref, sn_ref = _ORACLE_8K["ref"]
    check_outputs("o", to_np(o), o_ref, TOL_BF16)
    check_states("state", to_np(sout[0]), s_ref, TOL_BF16, (1, 2))
    check_states("snapshots", snaps.cpu().numpy(), sn_ref, TOL_BF16, (2, 3))


def test_ragged_prefix_resume(cuda_device):
    wl = synth.WORKLOADS["ragged_prefix_32"]
    plan = synth.ragged_plan(wl["seed"], wl["n_seq"], wl["mu"], wl["sigma"], wl["lo"], wl["hi"],
                             wl["prefix"], wl["n_resume"], wl["snap"])
    lens, start = plan["lens"], plan["start_pos"]
    n_seq, snap, P = len(lens), wl["snap"], wl["prefix"]
    # shared prefix: its own token stream (t0 = 0 of seed + 1); GPU snapshots every 256
    xp = synth.token_inputs(wl["seed"] + 1, P, H, D, D, io="bf16")
    devp = {k: v.to(cuda_device) for k, v in xp.items()}
    _, _, psnaps, _, _ = _prefill(devp, np.array([0, P], dtype=np.int32), snap=snap,
                                  device=cuda_device)
    # initial states: zero, or the prefix snapshot at the resume boundary (via kda_snapshot)
    s0 = torch.zeros((n_seq, H, D, D), device=cuda_device)
    res = plan["resumers"]
    src = torch.tensor([plan["resume_block"][s] - 1 for s in res], dtype=torch.int64,
                       device=cuda_device)
    dst = torch.tensor(res, dtype=torch.int64, device=cuda_device)
    K.kda_snapshot(src, dst, psnaps, s0)
    del devp
    # the packed batch
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = synth.token_inputs(wl["seed"], int(cu[-1]), H, D, D, io="bf16")
    dev = {k: v.to(cuda_device) for k, v in x.items()}
    o, sout, snaps, offs, pos = _prefill(dev, cu, start, s0, snap, cuda_device)
    # snapshot rows: exactly the planned absolute positions, per sequence
    for s in range(n_seq):
        want = [p for p in range(start[s] + 1, start[s] + lens[s] + 1) if p % snap == 0]
        assert pos[offs[s]:offs[s + 1]].tolist() == want
    heads = [0, 21, 42, 63]
    o_h = o[:, heads].float().cpu().numpy()
    s_h = sout[:, heads].cpu().numpy()
    sn_h = snaps[:, heads].cpu().numpy()
    for s in range(n_seq):
        a, b = int(cu[s]), int(cu[s + 1])
        seq = {k: v[a:b, heads] for k, v in x.items()}
        if start[s]:
            m = start[s]
            pre = {k: v[:m, heads] for k, v in xp.items()}
            seq = {k: torch.cat([pre[k], seq[k]]) for k in seq}
        ro, rs, rsn = native.oracle_sequence(seq["q"], seq["k"], seq["v"], seq["g"], seq["beta"],
                                             None, None, 0, snap, out_dtype=np.float32)
        ro = ro[start[s]:]
        rsn = rsn[start[s] // snap:]
        check_outputs(f"o seq {s}", o_h[a:b], ro, TOL_BF16)
        check_states(f"state seq {s}", s_h[s], rs, TOL_BF16, (1, 2))
        if len(rsn):
            check_states(f"snapshots seq {s}", sn_h[offs[s]:offs[s + 1]], rsn, TOL_BF16, (2, 3))


@pytest.mark.slow
def test_long_context_segments(cuda_device):
    wl = synth.WORKLOADS["long_1m"]
    T, seg, snap = wl["T"], wl["segment"], wl["snap"]
    heads = [0, 63]
    state = None
    o_keep, sn_keep, xs = [], [], {k: [] for k in ("q", "k", "v", "g", "beta")}
    for i in range(T // seg):
        x = synth.token_inputs(wl["seed"], seg, H, D, D, io="bf16", t0=i * seg)
        dev = {k: v.to(cuda_device) for k, v in x.items()}
        o, sout, snaps, offs, pos = _prefill(dev, np.array([0, seg], dtype=np.int32), [i * seg],
                                             state, snap, cuda_device)
        assert pos.tolist() == list(range(i * seg + snap, (i + 1) * seg + 1, snap))
        state = sout
        o_keep.append(o[:, heads].float().cpu().numpy())
        sn_keep.append(snaps[:, heads].cpu().numpy())
        for k in xs:
            xs[k].append(x[k][:, heads].clone())
        del dev, o, snaps
    xo = {k: torch.cat(v) for k, v in xs.items()}
    ro, rs, rsn = native.oracle_sequence(xo["q"], xo["k"], xo["v"], xo["g"], xo["beta"],
                                         None, None, 0, snap, out_dtype=np.float32)
    check_outputs("o", np.concatenate(o_keep), ro, TOL_BF16)
    check_states("state", state[0, heads].cpu().numpy(), rs, TOL_BF16, (1, 2))
    check_states("snapshots", np.concatenate(sn_keep), rsn, TOL_BF16, (2, 3))
