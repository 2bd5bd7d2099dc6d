"""Shared helpers of the GPU parity tests: seeded inputs (from synth), the
oracle's answers (from oracle/), and the tolerance metric.

Tolerance (stated for the KDA parity tests): max relative error, normwise per
(sequence, head) block, max|x - y| / max|y|, at most 2e-2 for bf16 q/k/v/o with
fp32 state, and 1e-4 when everything is fp32. Snapshot rows and cu_seqlens
handling are compared exactly.
"""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import native

TOL_BF16 = 2e-2
TOL_FP32 = 1e-4


def tol_for(io: str) -> float:
    return TOL_BF16 if io == "bf16" else TOL_FP32


def blockwise_err(x, ref, block_axes):
    """max over blocks of max|x - ref| / max|ref|; a block is one index of the
    axes NOT in block_axes (block_axes are reduced)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.max(np.abs(x - ref), axis=block_axes)
    den = np.max(np.abs(ref), axis=block_axes)
    bad = den == 0
    ratio = np.where(bad, num, num / np.where(bad, 1.0, den))
    return float(np.max(ratio)) if ratio.size else 0.0


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def packed_inputs(seed, lens, H, d, io, device):
    T = int(sum(lens))
    x = synth.token_inputs(seed, T, H, d, d, io=io)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    dev = {k: v.to(device) for k, v in x.items()}
    return x, dev, cu


def oracle_prefill(x, cu, start_pos=None, s0=None, snap=0):
    return native.oracle_packed(x["q"], x["k"], x["v"], x["g"], x["beta"], cu, start_pos,
                                s0, None, snap, out_dtype=np.float64)
