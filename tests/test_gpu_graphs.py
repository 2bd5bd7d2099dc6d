"""The serving calls inside a CUDA graph: a prefill (two launches through a
workspace), a decode step and a verify + commit step, captured once and replayed
on new inputs copied into the captured buffers, give the same bits as the same
calls made eagerly on those inputs. Each call is asynchronous on its stream,
allocates nothing, and takes its host arguments (sequence lengths) at capture,
so a serving loop can replay a step's launches without host work per launch.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from hybrid_linear_attention_04_b200 import kda as K

pytestmark = pytest.mark.gpu


def _inputs(seed, lens_p, n_seq, lens_prev, lens_draft, H, d):
    """One set of inputs for the three calls (CPU tensors)."""
    return {
        "p": synth.token_inputs(seed, int(sum(lens_p)), H, d, d, io="bf16"),
        "d": synth.token_inputs(seed + 1, n_seq, H, d, d, io="bf16"),
        "vp": synth.token_inputs(seed + 2, int(sum(lens_prev)), H, d, d, io="bf16"),
        "vc": synth.token_inputs(seed + 3, int(sum(lens_draft)), H, d, d, io="bf16"),
    }


def test_serving_step_replays_in_a_cuda_graph(cuda_device):
    H, d, n_seq = 8, 128, 16
    lens_p = [200, 77]
    cu_p = np.concatenate([[0], np.cumsum(lens_p)]).astype(np.int32)
    lens_prev = synth.draft_lengths(1600, n_seq, 1, 8)
    lens_draft = synth.draft_lengths(1601, n_seq, 1, 8)
    cp = np.concatenate([[0], np.cumsum(lens_prev)]).astype(np.int32)
    cd = np.concatenate([[0], np.cumsum(lens_draft)]).astype(np.int32)
    acc = [min(a, m) for a, m in zip(synth.randint(1600, "misc", n_seq, 0, 8), lens_prev)]
    pool0 = synth.states(1602, n_seq + 2, H, d, d, std=0.1).to(cuda_device)
    slots = torch.tensor(synth.permutation(1602, n_seq + 2, "slots")[:n_seq], dtype=torch.int32,
                         device=cuda_device)
    acc_d = torch.tensor(acc, dtype=torch.int32, device=cuda_device)

    # the captured (static) buffers
    set_a = _inputs(1610, lens_p, n_seq, lens_prev, lens_draft, H, d)
    set_b = _inputs(1620, lens_p, n_seq, lens_prev, lens_draft, H, d)
    buf = {g: {k: v.to(cuda_device) for k, v in x.items()} for g, x in set_a.items()}
    T = int(cu_p[-1])
    o_p = torch.empty((T, H, d), dtype=torch.bfloat16, device=cuda_device)
    s_p = torch.empty((len(lens_p), H, d, d), device=cuda_device)
    ws = torch.empty(K.kda_prefill_workspace_size(buf["p"]["q"], buf["p"]["v"], cu_p),
                     dtype=torch.uint8, device=cuda_device)
    o_d = torch.empty((n_seq, H, d), dtype=torch.bfloat16, device=cuda_device)
    o_v = torch.empty((int(cd[-1]), H, d), dtype=torch.bfloat16, device=cuda_device)
    pool = pool0.clone()

    def load(x):
        for g, t in x.items():
            for k, v in t.items():
                buf[g][k].copy_(v)
        pool.copy_(pool0)

    def step():
        p, dd, vp, vc = buf["p"], buf["d"], buf["vp"], buf["vc"]
        K.kda_prefill(p["q"], p["k"], p["v"], p["g"], p["beta"], cu_p, o_p, state_out=s_p,
                      chunk=64, workspace=ws)
        K.kda_decode(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], slots, pool, o_d)
        K.kda_verify_commit(vp, acc_d, cp, vc["q"], vc["k"], vc["v"], vc["g"], vc["beta"], cd,
                            slots, pool, o_v)

    def results():
        return [t.clone() for t in (o_p, s_p, o_d, o_v, pool)]

    # eager reference on set b
    load(set_b)
    step()
    torch.cuda.synchronize()
    assert K.kda_check_device_status() == 0
    ref = results()

    # capture on set a (after a warm-up on a side stream), replay on set b
    load(set_a)
    side = torch.cuda.Stream(device=cuda_device)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    n0 = K.kda_launch_count()
    with torch.cuda.graph(graph):
        step()
    captured = K.kda_launch_count() - n0
    assert captured >= 4                       # prep + chain, decode, verify + commit
    for t in (o_p, s_p, o_d, o_v):
        t.zero_()
    load(set_b)
    graph.replay()
    torch.cuda.synchronize()
    assert K.kda_check_device_status() == 0
    for name, a, b in zip(["prefill o", "prefill state", "decode o", "verify o", "pool"], results(),
                          ref):
        assert torch.equal(a, b), name
    # a second replay on set a gives set a's eager results, not set b's
    load(set_a)
    graph.replay()
    torch.cuda.synchronize()
    got_a = results()
    load(set_a)
    step()
    torch.cuda.synchronize()
    for a, b in zip(got_a, results()):
        assert torch.equal(a, b)
    del graph
