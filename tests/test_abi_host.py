"""Host-side tests of the C ABI (no GPU): the library loads, exports every
function include/kda.h declares, plans snapshots as the block-boundary rule
says (vLLM day-0 blog, "Kimi Delta Attention"), and rejects bad arguments
before anything is launched. Every call here fails validation or is host-only,
so no kernel is ever launched with the fake pointers these tests pass.
"""
from __future__ import annotations

import ctypes
import re
from pathlib import Path

import numpy as np
import pytest

import synth
from hybrid_linear_attention_04_b200 import build as kbuild
from hybrid_linear_attention_04_b200 import kda as K

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "kda.h"

# aligned and misaligned fake device addresses: never dereferenced, because
# every call that receives them fails validation on the host first.
A = ctypes.c_void_p(0x10000)
MIS = ctypes.c_void_p(0x10004)


@pytest.fixture(scope="module", autouse=True)
def built():
    kbuild.build()


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert {"kda_prefill", "kda_decode", "kda_verify", "kda_snapshot", "kda_snapshot_plan",
            "kda_check_device_status", "kda_status_string"} <= set(names)
    L = ctypes.CDLL(str(K.library_path()))
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    for code, name in K.STATUS_NAMES.items():
        assert K.kda_status_string(code).startswith(name)


def _plan_ref(cu, start, interval):
    offs, pos = [0], []
    for s in range(len(cu) - 1):
        p0, n = start[s], cu[s + 1] - cu[s]
        ps = [p for p in range(p0 + 1, p0 + n + 1) if interval and p % interval == 0]
        pos += ps
        offs.append(offs[-1] + len(ps))
    return offs, pos


@pytest.mark.parametrize("seed", range(6))
def test_snapshot_plan_matches_restatement(seed):
    n = 1 + seed * 7
    lens = synth.randint(seed, "lens", n, 0, 700)
    lens[0] = 0                                   # zero-length sequence
    if n > 2:
        lens[1] = 512                             # boundary-aligned end
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    start = [64 * m for m in synth.randint(seed, "resume", n, 0, 12)]
    for interval in (0, 64, 256):
        offs, pos = K.kda_snapshot_plan(cu, start, interval)
        ro, rp = _plan_ref(cu.tolist(), start, interval)
        assert offs.tolist() == ro
        assert pos.tolist() == rp


def test_snapshot_plan_rejects_bad_input():
    with pytest.raises(K.KDAError) as e:
        K.kda_snapshot_plan([1, 5], None, 4)
    assert e.value.status == 1
    with pytest.raises(K.KDAError):
        K.kda_snapshot_plan([0, 5, 3], None, 4)
    with pytest.raises(K.KDAError):
        K.kda_snapshot_plan([0, 5], [-1], 4)


def _dims(H=4, d=128, chunk=64, io=0, scale=0.0):
    return K.kda_dims(H, d, d, chunk, io, scale)


def _prefill(dims, cu, start=None, snap=0, ptr=A, snapshots=A, n_seq=None, ws=None, ws_bytes=0):
    cu = np.asarray(cu, dtype=np.int32)
    sp = None if start is None else np.asarray(start, dtype=np.int64)
    L = K.lib()
    return L.kda_prefill(ctypes.byref(dims), len(cu) - 1 if n_seq is None else n_seq,
                         cu.ctypes.data_as(ctypes.c_void_p),
                         None if sp is None else sp.ctypes.data_as(ctypes.c_void_p),
                         ptr, A, A, A, A, None, A, A, snap, snapshots, ws, ws_bytes, None)


def test_prefill_validation():
    assert _prefill(_dims(d=96), [0, 64]) == 2                 # unsupported head dim
    assert _prefill(K.kda_dims(4, 128, 64, 64, 0, 0.0), [0, 64]) == 2   # dk != dv
    assert _prefill(_dims(chunk=48), [0, 64]) == 2             # unsupported chunk
    assert _prefill(_dims(io=7), [0, 64]) == 1                 # bad io type
    assert _prefill(_dims(H=0), [0, 64]) == 1
    assert _prefill(_dims(), [0, 64], n_seq=-1) == 1
    assert _prefill(_dims(), [3, 64]) == 1                     # cu_seqlens[0] != 0
    assert _prefill(_dims(), [0, 64, 10]) == 1                 # decreasing
    assert _prefill(_dims(), [0, 300], snap=100) == 1          # interval % chunk != 0
    assert _prefill(_dims(), [0, 300], start=[32], snap=256) == 1   # start % chunk != 0
    assert _prefill(_dims(), [0, 300], start=[-64]) == 1
    assert _prefill(_dims(), [0, 300], snap=256, snapshots=None) == 1   # missing pool
    assert _prefill(_dims(), [0, 64], ptr=MIS) == 3            # misaligned q
    assert _prefill(_dims(), [0, 64], ptr=None) == 1           # null q
    assert _prefill(_dims(), [0], n_seq=0) == 0                # nothing to do
    need = _workspace_size(_dims(), [0, 64])
    assert _prefill(_dims(), [0, 64], ws=A, ws_bytes=need - 16) == 4   # workspace too small
    assert _prefill(_dims(), [0, 64], ws=MIS, ws_bytes=need) == 3      # misaligned workspace


def _workspace_size(dims, cu, n_seq=None):
    cu = np.asarray(cu, dtype=np.int32)
    n = ctypes.c_size_t(12345)
    st = K.lib().kda_prefill_workspace_size(ctypes.byref(dims), len(cu) - 1 if n_seq is None else n_seq,
                                            cu.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n))
    return n.value if st == 0 else -st


def test_prefill_workspace_size():
    """One packet of 75776 bytes per (64-token chunk row, head); chunk rows of a
    launch group are (group tokens >> 6) + group sequences, so that every
    sequence's ragged chunks get rows of their own."""
    P = 75776
    assert _workspace_size(_dims(H=4), [0, 64]) == (1 + 1) * 4 * P
    assert _workspace_size(_dims(H=2), [0, 1, 65, 200]) == ((200 >> 6) + 3) * 2 * P
    assert _workspace_size(_dims(H=1), [0], n_seq=0) == 0
    # more sequences than one launch: the largest group decides
    cu = np.arange(0, 64 * 1030 + 1, 64)
    assert _workspace_size(_dims(H=1), cu) == (1024 + 1024) * P
    # dimensions of the CUDA-core path use none
    assert _workspace_size(_dims(d=64, chunk=32), [0, 640]) == 0
    assert _workspace_size(_dims(io=1), [0, 640]) == 0
    # errors
    assert _workspace_size(_dims(), [0, 64, 10]) == -1
    assert _workspace_size(_dims(d=96), [0, 64]) == -2
    assert K.lib().kda_prefill_workspace_size(ctypes.byref(_dims()), 1,
                                              np.array([0, 64], np.int32).ctypes.data_as(ctypes.c_void_p),
                                              None) == 1


def test_decode_verify_snapshot_validation():
    L = K.lib()
    d = _dims()
    assert L.kda_decode(ctypes.byref(_dims(d=48)), 4, A, A, A, A, A, A, 8, A, A, None) == 2
    assert L.kda_decode(ctypes.byref(d), -1, A, A, A, A, A, A, 8, A, A, None) == 1
    assert L.kda_decode(ctypes.byref(d), 4, None, A, A, A, A, A, 8, A, A, None) == 1
    assert L.kda_decode(ctypes.byref(d), 4, A, A, A, A, A, MIS, 8, A, A, None) == 3
    assert L.kda_decode(ctypes.byref(d), 0, None, None, None, None, None, None, 0, None, None,
                        None) == 0
    cu = np.array([1, 3], dtype=np.int32)
    assert L.kda_verify(ctypes.byref(d), 1, cu.ctypes.data_as(ctypes.c_void_p), A, A, A, A, A, A,
                        8, A, A, A, None) == 1
    cu = np.array([0, 3, 2], dtype=np.int32)
    assert L.kda_verify(ctypes.byref(d), 2, cu.ctypes.data_as(ctypes.c_void_p), A, A, A, A, A, A,
                        8, A, A, A, None) == 1
    cu = np.array([0, 3], dtype=np.int32)
    assert L.kda_verify(ctypes.byref(d), 1, cu.ctypes.data_as(ctypes.c_void_p), A, A, A, A, A, A,
                        8, A, MIS, A, None) == 3
    assert L.kda_snapshot(-1, A, A, A, 4, A, 4, 4, 128, 128, None) == 1
    assert L.kda_snapshot(2, A, A, A, 4, A, 4, 1, 3, 1, None) == 2
    assert L.kda_snapshot(2, A, MIS, A, 4, A, 4, 4, 128, 128, None) == 3
    assert L.kda_snapshot(2, None, A, A, 4, A, 4, 4, 128, 128, None) == 1
    assert L.kda_snapshot(0, None, None, None, 0, None, 0, 4, 128, 128, None) == 0


def test_verify_commit_validation():
    L = K.lib()
    d = _dims()
    cu2 = np.array([0, 3, 5], dtype=np.int32)
    bad = np.array([0, 3, 2], dtype=np.int32)
    P = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731

    def call(dims=d, n=2, cp=cu2, cd=cu2, kp=A, na=A, pos=None, snap=0, srow=None, sn=None,
             q=A, slots=A, pool=A, o=A):
        return L.kda_verify_commit(ctypes.byref(dims), n, P(cp), kp, A, A, A, na, pos, snap, srow,
                                   sn, 0, P(cd), q, A, A, A, A, None, slots, 8, pool, o, None)
    assert call(dims=_dims(d=48)) == 2                   # unsupported head dim
    assert call(n=-1) == 1
    assert call(cp=bad) == 1 and call(cd=bad) == 1       # decreasing offsets
    assert call(kp=None) == 1                            # previous batch without its tensors
    assert call(na=None) == 1                            # acceptance counts are required
    assert call(q=None) == 1
    assert call(snap=256, srow=A) == 1                   # snapshot rows without positions
    assert call(o=MIS) == 3
    assert call(na=MIS) == 3
    assert call(n=0) == 0


def test_frontend_validation():
    L = K.lib()
    d = _dims()
    cu = np.array([0, 64, 100], dtype=np.int32)
    P = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    conv = K.kda_conv(4, 0x10000, 0x10000)
    bad_taps = K.kda_conv(5, 0x10000, 0x10000)
    no_w = K.kda_conv(4, None, 0x10000)
    mis_w = K.kda_conv(4, 0x10008, 0x10000)

    def fe(cv=conv, n=2, c=cu, snap=0, sn=None, qo=A, start=None):
        return L.kda_qk_frontend(ctypes.byref(d), None if cv is None else ctypes.byref(cv), n, P(c),
                                 start, A, A, None, None, qo, A, snap, sn, None)
    assert fe(cv=None) == 1 and fe(cv=bad_taps) == 1 and fe(cv=no_w) == 1
    assert fe(cv=mis_w) == 3
    assert fe(c=np.array([0, 64, 10], np.int32)) == 1
    assert fe(snap=96) == 1                        # not a multiple of the chunk
    assert fe(snap=64) == 1                        # snapshots due, no conv snapshot pool
    assert fe(qo=None) == 1 and fe(qo=MIS) == 3
    assert fe(n=0) == 0
    st = np.array([32, 0], dtype=np.int64)
    assert fe(snap=64, sn=A, start=P(st)) == 1     # start position off the chunk grid
    # decode / verify / verify+commit with the front-end
    assert L.kda_decode_conv(ctypes.byref(d), None, 4, A, A, A, A, A, A, 8, A, A, A, None) == 1
    assert L.kda_decode_conv(ctypes.byref(d), ctypes.byref(conv), 4, A, A, A, A, A, A, 8, A, None,
                             A, None) == 1         # no conv pool
    assert L.kda_decode_conv(ctypes.byref(d), ctypes.byref(bad_taps), 4, A, A, A, A, A, A, 8, A, A,
                             A, None) == 1
    c2 = np.array([0, 3, 5], dtype=np.int32)
    assert L.kda_verify_conv(ctypes.byref(d), ctypes.byref(conv), 2, P(c2), A, A, A, A, A, A, 8, A,
                             None, A, None, A, None) == 1
    assert L.kda_verify_conv(ctypes.byref(d), ctypes.byref(conv), 2, P(c2), A, A, A, A, A, A, 8, A,
                             A, A, MIS, A, None) == 3
    # verify+commit with the front-end needs the previous batch's raw q
    assert L.kda_verify_commit_conv(ctypes.byref(d), ctypes.byref(conv), 2, P(c2), None, A, A, A, A,
                                    A, None, 0, None, None, None, 0, P(c2), A, A, A, A, A, None, A,
                                    8, A, A, A, None) == 1


def test_no_launch_issued_by_host_tests():
    # the validation failures above must not have launched anything
    assert K.kda_launch_count() == 0


def test_binding_workspace_argument():
    """The binding's workspace argument: a wrong kind raises before any CUDA call, and
    its size query matches the C function for tensors of the prefill's shape."""
    import torch
    q = torch.zeros((200, 4, 128), dtype=torch.bfloat16)
    cu = [0, 70, 200]
    with pytest.raises(K.KDAError) as e:
        K.kda_prefill(q, q, q, q.float(), q[..., 0].float(), cu, q, workspace="bogus")
    assert e.value.status == 1
    assert K.kda_prefill_workspace_size(q, q, cu) == ((200 >> 6) + 2) * 4 * 75776
    assert K.kda_prefill_workspace_size(q.float(), q.float(), cu) == 0     # fp32 I/O: CUDA-core path


def test_workspace_rows_are_disjoint_and_within_the_reported_size():
    """Both prefill kernels place chunk c of sequence i (of a launch group whose first
    token is tok_first) at packet row ((tok0_i - tok_first) >> 6) + i + c. For random
    ragged batches those rows never collide and stay below the rows that
    kda_prefill_workspace_size reports for the group."""
    rng = np.random.default_rng(5)
    for trial in range(200):
        n = int(rng.integers(1, 40))
        lens = rng.integers(0, 400, size=n)
        lens[rng.random(n) < 0.2] = 0
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        H = int(rng.integers(1, 5))
        rows = set()
        for i in range(n):
            first = ((int(cu[i]) - 0) >> 6) + i
            for c in range((int(lens[i]) + 63) // 64):
                assert first + c not in rows
                rows.add(first + c)
        size = _workspace_size(_dims(H=H), cu)
        assert size % (H * 75776) == 0
        assert all(r < size // (H * 75776) for r in rows)
