"""The device input generator produces the host generator's bits."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("start,count", [(0, 100000), (123457, 5000), ((1 << 32) + 3, 777)])
def test_device_matches_host(start, count):
    out = torch.empty(count, dtype=torch.float32, device="cuda")
    synth.device_master(out, 0, 4, start)
    assert np.array_equal(out.cpu().numpy(), synth.master(0, 4, start, count))
    synth.device_m_warm(out, 0, 4, start)
    assert np.array_equal(out.cpu().numpy(), synth.m_warm(0, 4, start, count))
    synth.device_v_warm(out, 0, 4, start)
    assert np.array_equal(out.cpu().numpy(), synth.v_warm(0, 4, start, count))
    b = torch.empty(count, dtype=torch.int16, device="cuda")
    synth.device_grad(b, 0, 4, 3, start)
    assert np.array_equal(b.cpu().numpy().view(np.uint16), synth.grad_bits(0, 4, 3, start, count))
    synth.device_activations(b, 0, 4, start)
    assert np.array_equal(b.cpu().numpy().view(np.uint16), synth.activations_bits(0, 4, start, count))
    synth.device_weight(b, 0, 4, start)
    assert np.array_equal(b.cpu().numpy().view(np.uint16), synth.weight_bits(0, 4, start, count))


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_state_codes_device_matches_host(fmt):
    out = torch.empty(5000, dtype=torch.uint8, device="cuda")
    for signed in (False, True):
        synth.device_state_codes(out, 0, 3, 2, fmt, signed, 777)
        assert np.array_equal(out.cpu().numpy(), synth.state_codes(0, 3, 2, 777, 5000, fmt, signed))
