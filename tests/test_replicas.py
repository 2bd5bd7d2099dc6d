"""Host logic of the N > 1 benchmark path, on CPU with two gloo ranks.

The KDA layer has no exchange step, so N GPUs run N independent replicas; the
only cross-rank operations are the barrier and the max over ranks of the event
times, which these tests exercise with world_size 2 on the gloo backend.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import sys
    from pathlib import Path
    sys.path.insert(0, str(Path(__file__).resolve().parents[1]))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    local = [10.0 + rank, 3.0 - rank, 0.5]
    dist.barrier()
    got = bench.max_over_ranks(dist, local, torch.device("cpu"))
    # the reference arm runs on rank 0 only; other ranks return without work
    os.environ["RANK"] = str(rank)
    os.environ["WORLD_SIZE"] = str(world)
    ref = None
    if rank != 0:
        class A:
            steps, warmup, ref_tokens = 1, 3, 8
        ref = bench.run_reference(A())
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, ref))


def test_two_rank_max_over_ranks_and_reference_arm():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        rank, got, ref = q.get(timeout=120)
        out[rank] = (got, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        assert out[rank][0] == [11.0, 3.0, 0.5]       # element-wise max over the two ranks
    assert out[1][1] is None                          # non-zero rank: no reference work


def test_single_process_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(None, [1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]
