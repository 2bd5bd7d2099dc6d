"""Host logic of the context-parallel prefill on two gloo ranks (CPU): each rank
holds one segment's affine state map (computed here by the oracle, oracle/segments.py),
the maps are exchanged with torch.distributed all-gather, and each rank composes the
maps of the segments before its own into its entering state. The composition runs a
numpy stand-in for kda_state_map_apply (the GPU kernel is tested in
test_gpu_context_parallel.py). The entering states must equal the oracle's sequential
states at the segment boundaries."""
from __future__ import annotations

import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

import synth
from oracle import segments as SEG


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _maps(seed, T, H, d, world):
    x = synth.token_inputs(seed, T, H, d, d, io="fp32")
    L = T // world
    out = []
    for r in range(world):
        sl = slice(r * L, (r + 1) * L)
        Ms, Ns = [], []
        for h in range(H):
            m, n = SEG.segment_map(x["k"][sl, h].double().numpy(), x["v"][sl, h].double().numpy(),
                                   x["g"][sl, h].double().numpy(), x["beta"][sl, h].double().numpy())
            Ms.append(m)
            Ns.append(n)
        out.append((np.stack(Ms), np.stack(Ns)))
    return x, out


def _apply_np(m, xx, out, nn):
    out.copy_(torch.from_numpy(m.numpy() @ xx.numpy() + nn.numpy()))


def _worker(rank, world, port, seed, T, H, d, q):
    import torch.distributed as dist
    from hybrid_linear_attention_04_b200 import context_parallel as CP
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        _, maps = _maps(seed, T, H, d, world)
        m, n = (torch.from_numpy(a) for a in maps[rank])
        Ms, Ns = CP.exchange_maps(m, n)
        s0 = torch.from_numpy(np.full((H, d, d), 0.01))
        S = CP.entering_states(Ms, Ns, s0, apply=_apply_np)
        q.put((rank, S[rank].numpy()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_compose_entering_states():
    world, seed, T, H, d = 2, 77, 24, 2, 8
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seed, T, H, d, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # oracle: the state at each segment boundary, stepping token by token from s0
    x, maps = _maps(seed, T, H, d, world)
    S = np.full((H, d, d), 0.01)
    L = T // world
    for r in range(world):
        assert np.allclose(got[r], S, rtol=1e-12, atol=1e-12), r
        for h in range(H):
            for t in range(r * L, (r + 1) * L):
                A, B = SEG.step_map(x["k"][t, h].double().numpy(), x["v"][t, h].double().numpy(),
                                    x["g"][t, h].double().numpy(), float(x["beta"][t, h]))
                S[h] = A @ S[h] + B
