"""Failure detection without a GPU fault: a bounded device wait that runs out
reports KDA_ERR_TIMEOUT through the status word and leaves the context usable;
an injected launch failure surfaces as KDA_ERR_CUDA on the host."""
from __future__ import annotations

import pytest
import torch

import synth
from hybrid_linear_attention_04_b200 import kda as K

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_device):
    assert K.kda_check_device_status() == 0
    st = K.lib().kda_test_wait_timeout(50, None)       # ~50 polls of 1 us on a flag never set
    assert st == 0
    assert K.kda_check_device_status() == 6
    # the context is still usable: a real call succeeds afterwards
    x = synth.token_inputs(3, 2, 2, 32, 32, io="fp32")
    dev = {k: v.to(cuda_device) for k, v in x.items()}
    pool = synth.states(3, 2, 2, 32, 32).to(cuda_device)
    slots = torch.tensor([1, 0], dtype=torch.int32, device=cuda_device)
    o = torch.empty_like(dev["v"])
    K.kda_decode(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], slots, pool, o)
    assert K.kda_check_device_status() == 0


def test_injected_launch_failure_is_reported(cuda_device):
    x = synth.token_inputs(4, 2, 2, 32, 32, io="fp32")
    dev = {k: v.to(cuda_device) for k, v in x.items()}
    pool = synth.states(4, 2, 2, 32, 32).to(cuda_device)
    before = pool.clone()
    slots = torch.tensor([0, 1], dtype=torch.int32, device=cuda_device)
    o = torch.empty_like(dev["v"])
    K.lib().kda_test_fail_next_launches(1)
    with pytest.raises(K.KDAError) as e:
        K.kda_decode(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], slots, pool, o)
    assert e.value.status == 5
    torch.cuda.synchronize()
    assert torch.equal(pool, before)                    # nothing ran
    K.kda_decode(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], slots, pool, o)
    assert K.kda_check_device_status() == 0
    assert not torch.equal(pool, before)
