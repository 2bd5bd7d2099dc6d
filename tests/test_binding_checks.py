"""The binding's argument checks (host only, no GPU): a tensor of the wrong dtype, trailing
shape or too few rows for the call is rejected with KDAError status 1 before any device
pointer is taken, so that it cannot address memory outside its buffer on the device; a
well-formed call passes them and stops only at the device-tensor check (CPU tensors here)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from hybrid_linear_attention_04_b200 import kda as K

H, D = 2, 64


def _tok(T, io=torch.bfloat16):
    z = lambda *s, dt=io: torch.zeros(s, dtype=dt)  # noqa: E731
    return {"q": z(T, H, D), "k": z(T, H, D), "v": z(T, H, D), "g": z(T, H, D, dt=torch.float32),
            "beta": z(T, H, dt=torch.float32), "o": z(T, H, D)}


def _raises(fn, *words):
    with pytest.raises(K.KDAError) as e:
        fn()
    assert e.value.status == 1
    for w in words:
        assert w in str(e.value), (w, str(e.value))


def _prefill(x, cu, **kw):
    return lambda: K.kda_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], cu, x["o"],
                                 workspace=None, **kw)


def test_prefill_checks():
    cu = np.array([0, 70, 130], np.int32)
    x = _tok(130)
    _raises(_prefill(x, cu), "device tensor expected")              # well formed: passes the checks
    _raises(_prefill(_tok(129), cu), "q has 129 rows")
    y = dict(x, g=x["g"].bfloat16())
    _raises(_prefill(y, cu), "g must be torch.float32")
    y = dict(x, k=torch.zeros(130, H + 1, D, dtype=torch.bfloat16))
    _raises(_prefill(y, cu), "k must be shaped")
    y = dict(x, v=x["v"].float())
    _raises(_prefill(y, cu), "v must be torch.bfloat16")
    _raises(_prefill(x, cu, state_in=torch.zeros(1, H, D, D)), "state_in has 1 rows")
    _raises(_prefill(x, cu, start_pos=[0]), "start_pos has 1 entries")
    # snapshots every 64 tokens: 1 + 0 rows for the two sequences (70 and 60 tokens)
    _raises(_prefill(x, cu, snap_interval=64, snapshots=torch.zeros(0, H, D, D)), "snapshots has 0 rows")
    _raises(_prefill(x, cu, snap_interval=64), "snapshots is required")
    e = _tok(0)
    _raises(_prefill(e, np.zeros(3, np.int32)), "device tensor expected")   # no tokens: passes


def test_decode_and_verify_checks():
    x = _tok(5)
    pool = torch.zeros(7, H, D, D)
    slots = torch.zeros(5, dtype=torch.int32)
    dec = lambda **o: (lambda: K.kda_decode(*(o.get(n, x[n]) for n in ("q", "k", "v", "g", "beta")),  # noqa: E731
                                            o.get("slots", slots), o.get("pool", pool), x["o"]))
    _raises(dec(), "device tensor expected")
    _raises(dec(slots=slots.long()), "slots must be torch.int32")
    _raises(dec(slots=slots[:4]), "slots has 4 rows")
    _raises(dec(pool=torch.zeros(7, H, D, D + 1)), "state_pool must be shaped")
    _raises(dec(beta=torch.zeros(5, H, 1)), "beta must be shaped")
    cu = np.array([0, 2, 5], np.int32)
    ver = lambda ts: (lambda: K.kda_verify(x["q"], x["k"], x["v"], x["g"], x["beta"], cu,  # noqa: E731
                                           slots[:2], pool, ts, x["o"]))
    _raises(ver(torch.zeros(5, H, D, D)), "device tensor expected")
    _raises(ver(torch.zeros(4, H, D, D)), "token_states has 4 rows")


def test_verify_commit_and_conv_checks():
    n = 3
    cp, cd = np.array([0, 2, 3, 5], np.int32), np.array([0, 1, 3, 4], np.int32)
    prev, x = _tok(5), _tok(4)
    pool = torch.zeros(4, H, D, D)
    slots = torch.zeros(n, dtype=torch.int32)
    acc = torch.zeros(n, dtype=torch.int32)
    vc = lambda pv, **kw: (lambda: K.kda_verify_commit(pv, acc, cp, x["q"], x["k"], x["v"], x["g"],  # noqa: E731
                                                        x["beta"], cd, slots, pool, x["o"], **kw))
    _raises(vc(prev), "device tensor expected")
    _raises(vc(None), "prev k is required")
    _raises(vc(prev, commit_new=torch.zeros(n, dtype=torch.int32)), "commit_new must be torch.uint8")
    _raises(vc(prev, pos=torch.zeros(n, dtype=torch.int32)), "pos must be torch.int64")
    wq = torch.zeros(H, D, 4)
    cpool = torch.zeros(4, 2, H, D, 3)
    dcv = lambda cpl, w=wq: (lambda: K.kda_decode_conv(x["q"][:n], x["k"][:n], x["v"][:n],  # noqa: E731
                                                       x["g"][:n], x["beta"][:n], slots, pool,
                                                       cpl, x["o"][:n], w, w))
    _raises(dcv(cpool), "device tensor expected")
    _raises(dcv(cpool[:3]), "conv_pool has 3 rows")
    _raises(dcv(torch.zeros(4, 2, H, D, 2)), "conv_pool must be shaped")
    _raises(dcv(cpool, torch.zeros(H + 1, D, 4)), "conv weights")


def test_frontend_snapshot_and_state_map_checks():
    cu = np.array([0, 64], np.int32)
    q = torch.zeros(64, H, D, dtype=torch.bfloat16)
    w = torch.zeros(H, D, 4)
    fe = lambda qo, **kw: (lambda: K.kda_qk_frontend(q, q, w, w, cu, qo, q, **kw))  # noqa: E731
    _raises(fe(q), "device tensor expected")
    _raises(fe(q.float()), "q_out must be torch.bfloat16")
    _raises(fe(q, snap_interval=64, conv_snapshots=torch.zeros(0, 2, H, D, 3)), "conv_snapshots has 0 rows")
    src = torch.zeros(3, H, D, D)
    idx = torch.zeros(2, dtype=torch.int64)
    _raises(lambda: K.kda_snapshot(idx, idx, src, src), "device tensor expected")
    _raises(lambda: K.kda_snapshot(idx.int(), idx, src, src), "src_idx must be torch.int64")
    _raises(lambda: K.kda_snapshot(idx, idx, src, torch.zeros(3, H, D, D + 1)), "dst must be shaped")
    M = torch.zeros(2, D, D)
    _raises(lambda: K.kda_state_map_apply(M, torch.zeros(2, D, D), torch.zeros(2, D, D).double()),
            "must be fp32")
