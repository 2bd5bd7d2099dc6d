"""Context-parallel prefill of one long sequence across workers (one GPU each).

Each step of the KDA recurrence is affine in the state (see kda_state_map_apply in
include/kda.h), so a segment of the sequence maps the state entering it to the
state leaving it as S -> M S + N. A worker holding segment r of P:
  1. computes its map with two kda_prefill calls on its own tokens: N from the
     zero state, M from the identity state with v = 0 (dv = dk);
  2. exchanges maps with the other workers (one all-gather of 2 x H x dk x dk fp32
     per worker through torch.distributed: NCCL between GPUs);
  3. applies the maps of segments 0..r-1 to the sequence's initial state with
     kda_state_map_apply, which gives the state entering its segment;
  4. runs kda_prefill of its segment from that state (outputs, snapshots at the
     sequence's absolute positions, final state).
Every arithmetic step runs in libkda's kernels; this module moves tensors and
orders the calls. The same steps on one GPU, with the segments of one call as the
sequences of a packed batch, are `prefill_segments_on_one_device`.
"""
from __future__ import annotations

import numpy as np
import torch

from . import kda as K


def _identity_states(n, H, d, device):
    eye = torch.eye(d, dtype=torch.float32, device=device)
    return eye.expand(n, H, d, d).contiguous()


def segment_maps(q, k, v, g, beta, cu_seqlens, chunk=64, workspace="auto"):
    """Maps (M, N) [n_seg, H, dk, dk] of the segments of a packed batch (each sequence
    of cu_seqlens one segment): N = final state from zero, M = final state with v = 0
    from the identity state."""
    cu = np.asarray(cu_seqlens, dtype=np.int32)
    n, H, d = len(cu) - 1, q.shape[1], q.shape[2]
    if v.shape[2] != d:
        raise K.KDAError(2, "segment maps need dv == dk")
    o = torch.empty_like(v)
    N = torch.empty((n, H, d, d), dtype=torch.float32, device=q.device)
    M = torch.empty_like(N)
    K.kda_prefill(q, k, v, g, beta, cu, o, state_out=N, chunk=chunk, workspace=workspace)
    K.kda_prefill(q, k, torch.zeros_like(v), g, beta, cu, o, state_out=M,
                  state_in=_identity_states(n, H, d, q.device), chunk=chunk, workspace=workspace)
    return M, N


def entering_states(M, N, S0=None, apply=None):
    """The state entering each segment: S_0 = S0 (zeros if None), S_{j+1} = M_j S_j + N_j.
    M, N [P, H, dk, dk]; returns [P, H, dk, dk]. `apply(M, X, out, N)` computes
    out = M X + N per head (kda_state_map_apply unless given)."""
    apply = apply or (lambda m, x, out, nn: K.kda_state_map_apply(m, x, out, N=nn))
    P = M.shape[0]
    out = torch.empty_like(N)
    out[0] = 0.0 if S0 is None else S0
    for j in range(P - 1):
        apply(M[j], out[j], out[j + 1], N[j])
    return out


def prefill_segments_on_one_device(q, k, v, g, beta, seg_len, state_in=None, start_pos=0,
                                   snap_interval=0, chunk=64, workspace="auto"):
    """One sequence of T = P * seg_len tokens processed as P segments whose maps are
    computed independently, composed, and then used to run every segment from its
    entering state: the arithmetic of the context-parallel prefill on one device.
    Returns (o [T, H, dv], final state [H, dk, dv], snapshots)."""
    T, H, d = q.shape
    if T % seg_len or seg_len % chunk or (snap_interval and seg_len % snap_interval):
        raise K.KDAError(1, "segments must be whole chunks and whole snapshot blocks")
    P = T // seg_len
    cu = np.arange(P + 1, dtype=np.int32) * seg_len
    M, N = segment_maps(q, k, v, g, beta, cu, chunk, workspace)
    S = entering_states(M, N, None if state_in is None else state_in.reshape(H, d, d))
    starts = [start_pos + j * seg_len for j in range(P)]
    offs, _ = K.kda_snapshot_plan(cu, starts, snap_interval)
    o = torch.empty_like(v)
    fin = torch.empty((P, H, d, d), dtype=torch.float32, device=q.device)
    snaps = torch.empty((int(offs[-1]), H, d, d), dtype=torch.float32, device=q.device)
    K.kda_prefill(q, k, v, g, beta, cu, o, state_out=fin, state_in=S, start_pos=starts,
                  snap_interval=snap_interval, snapshots=snaps, chunk=chunk, workspace=workspace)
    return o, fin[P - 1], snaps


def exchange_maps(M, N, group=None, dist=None):
    """All-gather one worker's map (M, N) [H, dk, dk] into [world, H, dk, dk] each."""
    if dist is None:
        import torch.distributed as dist
    world = dist.get_world_size(group)
    Ms = [torch.empty_like(M) for _ in range(world)]
    Ns = [torch.empty_like(N) for _ in range(world)]
    dist.all_gather(Ms, M.contiguous(), group=group)
    dist.all_gather(Ns, N.contiguous(), group=group)
    return torch.stack(Ms), torch.stack(Ns)


def context_parallel_prefill(q, k, v, g, beta, rank, seg_start, state_in=None,
                             snap_interval=0, chunk=64, workspace="auto", group=None,
                             apply=None):
    """This worker's part of a context-parallel prefill: its segment's tokens
    (q, k, v, g, beta [L, H, d]) starting at absolute position seg_start, the
    sequence's initial state (on every worker; None = zeros). Returns (o, final
    state of this segment [H, dk, dv], its snapshots)."""
    L, H, d = q.shape
    cu = np.array([0, L], dtype=np.int32)
    M, N = segment_maps(q, k, v, g, beta, cu, chunk, workspace)
    Ms, Ns = exchange_maps(M[0], N[0], group)
    S = entering_states(Ms, Ns, state_in, apply)[rank]
    offs, _ = K.kda_snapshot_plan(cu, [seg_start], snap_interval)
    o = torch.empty_like(v)
    fin = torch.empty((1, H, d, d), dtype=torch.float32, device=q.device)
    snaps = torch.empty((int(offs[-1]), H, d, d), dtype=torch.float32, device=q.device)
    K.kda_prefill(q, k, v, g, beta, cu, o, state_out=fin, state_in=S[None].contiguous(),
                  start_pos=[seg_start], snap_interval=snap_interval, snapshots=snaps,
                  chunk=chunk, workspace=workspace)
    return o, fin[0], snaps
