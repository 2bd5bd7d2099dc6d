"""The seeded input generator: the device-side drawing (used for the benchmark's
largest inputs) produces the same streams as the host-side one."""
from __future__ import annotations

import numpy as np
import torch

import synth


def test_device_generator_matches_host_streams():
    x = synth.token_inputs(1003, 130, 3, 64, 64, io="bf16", t0=501)
    y = synth.token_inputs_device(1003, 130, 3, 64, 64, io="bf16", t0=501, device="cpu")
    for k in x:
        assert torch.equal(x[k], y[k]), k
    s1 = synth.states(9, 2, 3, 16, 16, std=0.1)
    s2 = synth.states_device(9, 2, 3, 16, 16, std=0.1, device="cpu")
    assert torch.equal(s1, s2)


def test_device_generator_laws():
    y = synth.token_inputs_device(7, 2000, 2, 128, 128, io="fp32", device="cpu")
    n = torch.linalg.vector_norm(y["q"].double(), dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-6)
    assert 0.0 < float(y["beta"].min()) and float(y["beta"].max()) < 1.0
    assert float(y["g"].max()) < 0.0
    v = y["v"].double().flatten()
    assert abs(float(v.mean())) < 0.01 and abs(float(v.std()) - 1.0) < 0.01
