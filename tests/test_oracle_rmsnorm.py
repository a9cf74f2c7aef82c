"""Pins for the oracle's FP8 RMSNorm layer (x / sqrt(mean(x^2) + eps) * w on
FP8 1x128 input, FP8 1x128 output; bf16 gradients dx and the weight gradient
dw from the saved FP8 input).

Pinned to a hand case (a row of one magnitude), to the composition of the
separately pinned codec functions with torch's rms_norm in float64 (a library
routine), and the backward to torch autograd on the dequantised input."""
import math

import numpy as np
import pytest
import torch

import synth

E4M3, E5M2 = 0, 1
EPS = 1e-6


def _bf16_of_f64(x):
    t = torch.from_numpy(np.asarray(x, np.float64)).to(torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _f64_of_bf16(bits):
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16) \
        .to(torch.float64).numpy()


def _inputs(orc, rows, d, fmt, expand_in, seed):
    x = synth.bf16_bits_to_f32(synth.activations_bits(seed, 0, 0, rows * d)).reshape(rows, d)
    xa = orc.group_quantize(x.astype(np.float64), 1, 128, expand_in, fmt)
    w = _bf16_of_f64(1.0 + 0.1 * synth.bf16_bits_to_f32(synth.weight_bits(seed, 1, 0, d)) / 0.02)
    return xa, w


def test_hand_case_one_magnitude(orc):
    """Every x = +-2 (code 0x40 = 2 in E4M3, scale 1, k 1), w = 1: mean(x^2) = 4,
    rstd = 1 / sqrt(4 + eps), y = +-2 rstd; the output group max is 2 rstd, so
    without expansion every code is +-448 and the root scale is 2 rstd / 448."""
    rows, d = 2, 256
    q = np.full((rows, d), 0x40, np.uint8)
    q[:, 1::2] |= 0x80
    one = np.ones((rows, 2), np.float32)
    w = _bf16_of_f64(np.ones(d))
    (oq, os_, ok), rstd = orc.rmsnorm_fp8_forward((q, one, one), w, EPS, E4M3, False,
                                                  want_rstd=True)
    assert np.all(rstd == 1.0 / math.sqrt(4.0 + EPS))
    assert np.all(oq[:, ::2] == 0x7E) and np.all(oq[:, 1::2] == 0xFE)
    assert np.all(os_ == np.float32(2.0 * rstd[0] / 448.0))
    assert np.all(ok == 1.0)
    # backward with dy = 1: g = 1, mean(g xh) = mean(xh) = 0 (signs alternate), so
    # dx = rstd; dw = sum over rows of xh = 2 rows * (+-2 rstd)
    dy = _bf16_of_f64(np.ones((rows, d)))
    dx, dw = orc.rmsnorm_fp8_backward(dy, (q, one, one), w, EPS, E4M3)
    assert np.array_equal(dx, _bf16_of_f64(np.full((rows, d), rstd[0])))
    assert np.allclose(dw[::2], 4.0 * rstd[0], rtol=1e-15)
    assert np.allclose(dw[1::2], -4.0 * rstd[0], rtol=1e-15)


@pytest.mark.parametrize("fmt,expand_in,expand_out", [(E4M3, False, False), (E4M3, True, True),
                                                      (E5M2, False, True)])
def test_forward_is_the_composition_of_the_codec_and_torch_rms_norm(orc, fmt, expand_in,
                                                                     expand_out):
    rows, d = 6, 640
    xa, w = _inputs(orc, rows, d, fmt, expand_in, 3)
    got, rstd = orc.rmsnorm_fp8_forward(xa, w, EPS, fmt, expand_out, want_rstd=True)
    x = torch.from_numpy(orc.group_dequantize(*xa, 1, 128, fmt))
    wt = torch.from_numpy(_f64_of_bf16(w))
    y = torch.nn.functional.rms_norm(x, (d,), wt, eps=EPS).numpy()
    want = orc.group_quantize(y, 1, 128, expand_out, fmt)
    for a, b in zip(got, want):
        assert np.array_equal(a, b)
    ref_rstd = 1.0 / np.sqrt((x.numpy() ** 2).mean(axis=1) + EPS)
    assert np.allclose(rstd, ref_rstd, rtol=1e-14)


@pytest.mark.parametrize("fmt,expand_in", [(E4M3, False), (E4M3, True), (E5M2, False)])
def test_backward_matches_autograd_on_the_dequantised_input(orc, fmt, expand_in):
    rows, d = 5, 384
    xa, w = _inputs(orc, rows, d, fmt, expand_in, 4)
    dy = synth.grad_bits(4, 2, 1, 0, rows * d).reshape(rows, d)
    dx, dw = orc.rmsnorm_fp8_backward(dy, xa, w, EPS, fmt)
    x = torch.tensor(orc.group_dequantize(*xa, 1, 128, fmt), requires_grad=True)
    wt = torch.tensor(_f64_of_bf16(w), requires_grad=True)
    torch.nn.functional.rms_norm(x, (d,), wt, eps=EPS).backward(torch.from_numpy(_f64_of_bf16(dy)))
    assert np.array_equal(dx, _bf16_of_f64(x.grad.numpy()))
    assert np.allclose(dw, wt.grad.numpy(), rtol=1e-12, atol=0)
