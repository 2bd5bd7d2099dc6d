"""ctypes loader for the C fp64 oracle (kda_oracle.c).

TEST INFRASTRUCTURE (see the package docstring). Building this library is part
of ``__graft_entry__.build()`` (building the checker is not using it).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np
import torch

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "kda_oracle.c"
_LIB = _HERE / "_kda_oracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile kda_oracle.c with gcc (-O2, OpenMP) into oracle/_kda_oracle.so."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                        str(_SRC), "-o", str(tmp), "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB))
        f = lib.kda_oracle_sequence
        f.restype = ctypes.c_int64
        f.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_double,
                      ctypes.c_int64,
                      ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                      ctypes.c_int, ctypes.c_int]
        lib.kda_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(load().kda_oracle_max_threads())


def _f32(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu", torch.float32).contiguous().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def oracle_sequence(q, k, v, g, beta, s0=None, scale=None, start_pos=0, snap_interval=0,
                    out_dtype=np.float64, n_threads=0):
    """Run the C oracle on one sequence (all heads).

    q, k, g: [T, H, dk]; v: [T, H, dv]; beta: [T, H]; s0: [H, dk, dv] or None.
    Inputs are passed as fp32 (bf16 and fp32 values are exact in fp32); an fp64
    numpy s0 is passed as fp64 (resuming from the oracle's own snapshot);
    arithmetic is fp64. Returns (o [T,H,dv], s_final [H,dk,dv], snaps [n,H,dk,dv]).
    """
    lib = load()
    s0_f64 = isinstance(s0, np.ndarray) and s0.dtype == np.float64
    if s0_f64:
        s0 = np.ascontiguousarray(s0)
    else:
        s0 = _f32(s0)
    q, k, v, g, beta = (_f32(x) for x in (q, k, v, g, beta))
    T, H, dk = k.shape
    dv = v.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    n_snap = 0
    if snap_interval > 0:
        n_snap = (start_pos + T) // snap_interval - start_pos // snap_interval
    o = np.empty((T, H, dv), dtype=out_dtype)
    sf = np.empty((H, dk, dv), dtype=out_dtype)
    sn = np.empty((n_snap, H, dk, dv), dtype=out_dtype)
    got = lib.kda_oracle_sequence(T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                  _ptr(s0), int(s0_f64), float(scale), int(start_pos),
                                  int(snap_interval),
                                  _ptr(o), _ptr(sf), _ptr(sn) if n_snap else None,
                                  int(out_dtype == np.float32), int(n_threads))
    assert got == n_snap
    return o, sf, sn


def oracle_packed(q, k, v, g, beta, cu_seqlens, start_pos=None, s0=None, scale=None,
                  snap_interval=0, out_dtype=np.float64, n_threads=0):
    """The C oracle over a packed ragged batch: sequence s is tokens
    [cu_seqlens[s], cu_seqlens[s+1]); s0 is [n_seq, H, dk, dv] or None.
    Returns (o [T_total,H,dv], s_final [n_seq,H,dk,dv], snaps [n_total,H,dk,dv])
    with the snapshots of sequence 0 first, each sequence's in ascending position.
    """
    n_seq = len(cu_seqlens) - 1
    start_pos = [0] * n_seq if start_pos is None else list(start_pos)
    outs, finals, snaps = [], [], []
    for s in range(n_seq):
        a, b = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        o, sf, sn = oracle_sequence(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b],
                                    None if s0 is None else s0[s], scale, start_pos[s],
                                    snap_interval, out_dtype, n_threads)
        outs.append(o)
        finals.append(sf)
        snaps.append(sn)
    return np.concatenate(outs), np.stack(finals), np.concatenate(snaps)
