"""GPU parity of the context-parallel prefill arithmetic (one long sequence split
into segments whose affine state maps are computed independently and composed;
runtimewire, "The architecture is built around inference cost": 1M-token context on a
fixed-size state), through the C ABI, against oracle/segments.py and the fp64 token
recurrence."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from hybrid_linear_attention_04_b200 import context_parallel as CP
from hybrid_linear_attention_04_b200 import kda as K
from kda_cases import TOL_BF16, check_outputs, check_states, to_np
from oracle import native
from oracle import segments as SEG

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (32, 64)])
def test_state_map_apply_matches_float64(cuda_device, dk, dv):
    rng = np.random.default_rng(dk + dv)
    n = 7
    M = rng.standard_normal((n, dk, dk)) / np.sqrt(dk)
    X = rng.standard_normal((n, dk, dv))
    N = rng.standard_normal((n, dk, dv))
    dev = lambda a: torch.from_numpy(a).float().to(cuda_device)  # noqa: E731
    out = torch.empty((n, dk, dv), device=cuda_device)
    Md, Xd, Nd = dev(M), dev(X), dev(N)
    K.kda_state_map_apply(Md, Xd, out, N=Nd)
    ref = M.astype(np.float32).astype(np.float64) @ X.astype(np.float32) + N.astype(np.float32)
    assert np.max(np.abs(to_np(out) - ref)) <= 1e-5 * np.max(np.abs(ref))
    K.kda_state_map_apply(Md, Xd, Nd, N=Nd)                   # out aliasing N
    assert torch.equal(Nd, out)
    assert K.kda_check_device_status() == 0


def test_segment_maps_match_oracle(cuda_device):
    """M (identity state, v = 0) and N (zero state) of a 200-token segment against the
    oracle's explicit product of the step maps."""
    H, d, L = 2, 128, 200
    x = synth.token_inputs(810, L, H, d, d, io="bf16")
    xd = {k: v.to(cuda_device) for k, v in x.items()}
    M, N = CP.segment_maps(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], [0, L])
    assert K.kda_check_device_status() == 0
    for h in range(H):
        m, nn = SEG.segment_map(x["k"][:, h].double().numpy(), x["v"][:, h].double().numpy(),
                                x["g"][:, h].double().numpy(), x["beta"][:, h].double().numpy())
        check_states("M", to_np(M[0, h])[None], m[None], TOL_BF16, (1, 2))
        check_states("N", to_np(N[0, h])[None], nn[None], TOL_BF16, (1, 2))


@pytest.mark.parametrize("path", ["split", "fused"])
def test_segments_on_one_device_equal_oracle(cuda_device, path):
    """4 segments of 512 tokens composed through their maps give the outputs, final
    state and snapshots of the one-pass oracle run (from an initial state, with the
    sequence's absolute snapshot positions)."""
    H, d, seg, P, snap = 4, 128, 512, 4, 256
    T = seg * P
    x = synth.token_inputs(820, T, H, d, d, io="bf16")
    s0 = synth.states(821, 1, H, d, d, std=0.1)
    xd = {k: v.to(cuda_device) for k, v in x.items()}
    ws = "auto" if path == "split" else None
    o, fin, snaps = CP.prefill_segments_on_one_device(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"],
                                                      seg, state_in=s0.to(cuda_device),
                                                      start_pos=1024, snap_interval=snap,
                                                      workspace=ws)
    assert K.kda_check_device_status() == 0
    o_ref, s_ref, sn_ref = native.oracle_sequence(x["q"], x["k"], x["v"], x["g"], x["beta"], s0[0],
                                                  None, 1024, snap)
    check_outputs("o", to_np(o), o_ref, TOL_BF16)
    check_states("state", to_np(fin)[None], s_ref[None], TOL_BF16, (2, 3))
    check_states("snapshots", snaps.cpu().numpy(), sn_ref, TOL_BF16, (2, 3))
