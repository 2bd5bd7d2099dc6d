"""Shared helpers of the GPU parity tests: seeded inputs (from synth), the
oracle's answers (from oracle/), and the tolerance metrics.

Tolerance (stated for the KDA parity tests): 2e-2 for bf16 q/k/v/o with fp32
state, 1e-4 when everything is fp32. Three measures of one result x against the
oracle's y are taken on every (sequence, head) block:
  normwise   max|x - y| / max|y| over the block (states, snapshots, outputs);
  per row    for outputs, every (token, head) row over d_v:
             max_row|x - y| / max(max_row|y|, 1e-3 * max_block|y|);
  elementwise |x - y| / (|y| + 1e-3 * max_block|y|), reported (not gated: bf16
             rounding of sums that cancel exceeds it by design) with the worst
             element's (token, head, column).
The normwise and per-row measures must both be within the tolerance. Snapshot
rows and cu_seqlens handling are compared exactly.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import synth
from oracle import native

TOL_BF16 = 2e-2
TOL_FP32 = 1e-4
FLOOR = 1e-3

# (test id, quantity, normwise, per-row, elementwise, worst element) of every checked result;
# written as JSON to $KDA_PARITY_REPORT at the end of the session when that is set
REPORT: list[dict] = []


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


def output_errors(x, ref, cu=None):
    """The three measures for outputs [T, H, d] of a packed batch (cu delimits the
    sequences; None = one sequence). Returns a dict with normwise, rowwise and
    elementwise maxima and the (token, head, column) of the worst element and of the
    worst row."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    T = x.shape[0]
    cu = [0, T] if cu is None else [int(c) for c in cu]
    out = {"normwise": 0.0, "rowwise": 0.0, "elementwise": 0.0, "worst_row": None,
           "worst_element": None}
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b <= a:
            continue
        xs, ys = x[a:b], ref[a:b]
        diff = np.abs(xs - ys)
        bmax = np.max(np.abs(ys), axis=(0, 2))                       # [H]
        norm = np.max(diff, axis=(0, 2)) / np.where(bmax > 0, bmax, 1.0)
        floor = FLOOR * bmax[None, :]                                # [1, H]
        rmax = np.max(np.abs(ys), axis=2)                            # [t, H]
        rden = np.maximum(rmax, floor)
        rerr = np.max(diff, axis=2) / np.where(rden > 0, rden, 1.0)
        eden = np.abs(ys) + floor[:, :, None]
        eerr = diff / np.where(eden > 0, eden, 1.0)
        out["normwise"] = max(out["normwise"], float(norm.max()))
        if float(rerr.max()) >= out["rowwise"]:
            t, h = np.unravel_index(int(np.argmax(rerr)), rerr.shape)
            out["rowwise"] = float(rerr.max())
            out["worst_row"] = (a + int(t), int(h))
        if float(eerr.max()) >= out["elementwise"]:
            t, h, c = np.unravel_index(int(np.argmax(eerr)), eerr.shape)
            out["elementwise"] = float(eerr.max())
            out["worst_element"] = (a + int(t), int(h), int(c))
    return out


def check_outputs(name, x, ref, tol, cu=None):
    """Assert the normwise and per-row measures of outputs against `tol` and record
    all three in REPORT."""
    e = output_errors(x, ref, cu)
    REPORT.append({"case": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0],
                   "quantity": name, "tol": tol, **e})
    assert e["normwise"] <= tol, (name, e)
    assert e["rowwise"] <= tol, (name, e)
    return e


def check_states(name, x, ref, tol, block_axes):
    """Assert the normwise measure of states or snapshots (blocks over block_axes) and
    record the elementwise-with-floor measure in REPORT."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    norm = blockwise_err(x, ref, block_axes)
    if ref.size:
        bmax = np.max(np.abs(ref), axis=block_axes, keepdims=True)
        eerr = float(np.max(np.abs(x - ref) / (np.abs(ref) + FLOOR * bmax + 1e-300)))
    else:
        eerr = 0.0
    REPORT.append({"case": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0],
                   "quantity": name, "tol": tol, "normwise": norm, "elementwise": eerr})
    assert norm <= tol, (name, norm)
    return norm


# Two GPU calls that run the same step: bit for bit (exact), or, for paths whose
# arithmetic differs, within fp32-level error.
SAME_STATE = 3e-5     # normwise per (slot, head) state


def same_states(a: torch.Tensor, b: torch.Tensor, exact: bool) -> bool:
    if exact:
        return torch.equal(a, b)
    x, y = a.double().cpu(), b.double().cpu()
    if not (torch.isfinite(x).all() and torch.isfinite(y).all()):
        return False
    diff = (x - y).flatten(-2).norm(dim=-1)
    ref = y.flatten(-2).norm(dim=-1)
    return bool((diff <= SAME_STATE * ref + 1e-30).all())


def same_outputs(a: torch.Tensor, b: torch.Tensor, exact: bool) -> bool:
    """bf16 outputs: one rounding step apart at most (2^-7 relative), plus a floor of
    1e-3 of the largest output for values near zero."""
    if exact:
        return torch.equal(a, b)
    x, y = a.double().cpu(), b.double().cpu()
    floor = 1e-3 * float(y.abs().max()) if y.numel() else 0.0
    return bool(((x - y).abs() <= 2.0 ** -7 * y.abs() + floor).all())


def write_report():
    path = os.environ.get("KDA_PARITY_REPORT")
    if path and REPORT:
        with open(path, "w") as f:
            json.dump(REPORT, f, indent=1)


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
