"""Pins for the oracle's FP8 SwiGLU layer (silu(gate) * up on FP8 1x128 inputs,
FP8 output, bf16 gradients from the saved FP8 inputs).

The activation and its derivatives are pinned to closed forms, to torch's
silu and autograd in float64 (library routines) and to finite differences;
the FP8 forward to a hand case whose output codes are the input codes and to
the composition of the separately pinned codec pieces; the backward to a
hand case and to autograd on the dequantised inputs."""
import math

import numpy as np
import pytest
import torch

import synth

E4M3, E5M2 = 0, 1


def _bf16_of_f64(x):
    """double -> FP32 -> bf16 bits, each rounding to nearest even (torch casts)."""
    t = torch.from_numpy(np.asarray(x, np.float64)).to(torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _f64_of_bf16(bits):
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16) \
        .to(torch.float64).numpy()


def test_swiglu_closed_forms(orc):
    assert orc.swiglu(0.0, 3.0) == 0.0
    assert orc.swiglu(1.7, 0.0) == 0.0
    # sigmoid(ln 3) = 3/4
    assert math.isclose(orc.swiglu(math.log(3.0), 1.0), 0.75 * math.log(3.0), rel_tol=1e-15)
    assert math.isclose(orc.swiglu(math.log(3.0), -2.0), -1.5 * math.log(3.0), rel_tol=1e-15)
    # e^-64 is below half an ulp of 1: sigmoid(64) is exactly 1 in double
    assert orc.swiglu(64.0, 5.0) == 320.0
    assert math.isclose(orc.swiglu(-64.0, 1.0), -64.0 * math.exp(-64.0), rel_tol=1e-12)
    # a sigmoid below FP32's normal range (2^-126) counts as 0
    assert orc.swiglu(-87.0, 1.0) != 0.0 and orc.swiglu(-88.0, 1.0) == 0.0
    assert orc.swiglu_grad(-88.0, 2.0, 1.0) == (0.0, 0.0)


def test_swiglu_grad_closed_forms(orc):
    assert orc.swiglu_grad(0.0, 2.0, 3.0) == (3.0, 0.0)        # sigmoid(0) = 1/2
    g = math.log(3.0)
    dg, du = orc.swiglu_grad(g, 2.0, 0.5)
    assert math.isclose(du, 0.5 * 0.75 * g, rel_tol=1e-15)
    assert math.isclose(dg, 0.5 * 2.0 * 0.75 * (1.0 + g / 4.0), rel_tol=1e-15)
    assert orc.swiglu_grad(64.0, -3.0, 2.0) == (-6.0, 128.0)


def test_swiglu_matches_torch_and_finite_differences(orc):
    rng = np.random.default_rng(7)
    g = np.concatenate([rng.normal(0, 3, 400), [-30.0, -5.0, -1e-3, 0.0, 1e-3, 5.0, 30.0]])
    u = rng.normal(0, 2, g.size)
    dh = rng.normal(0, 1, g.size)
    gt = torch.tensor(g, dtype=torch.float64, requires_grad=True)
    ut = torch.tensor(u, dtype=torch.float64, requires_grad=True)
    h = torch.nn.functional.silu(gt) * ut
    h.backward(torch.tensor(dh, dtype=torch.float64))
    for i in range(g.size):
        assert math.isclose(orc.swiglu(g[i], u[i]), h[i].item(), rel_tol=1e-14, abs_tol=1e-300)
        dg, du = orc.swiglu_grad(g[i], u[i], dh[i])
        assert math.isclose(dg, gt.grad[i].item(), rel_tol=1e-12, abs_tol=1e-15)
        assert math.isclose(du, ut.grad[i].item(), rel_tol=1e-12, abs_tol=1e-15)
        # central differences of the forward (independent of the derivative formula)
        e = 1e-5 * max(1.0, abs(g[i]))
        fd_g = dh[i] * (orc.swiglu(g[i] + e, u[i]) - orc.swiglu(g[i] - e, u[i])) / (2 * e)
        fd_u = dh[i] * (orc.swiglu(g[i], u[i] + 1e-5) - orc.swiglu(g[i], u[i] - 1e-5)) / 2e-5
        assert abs(dg - fd_g) <= 1e-6 * (1 + abs(dg))
        assert abs(du - fd_u) <= 1e-6 * (1 + abs(du))


def _inputs(rows, cols, fmt, seed, k_one=True):
    """FP8 gate/up drawn by the seeded generator: codes over the format's range
    with random signs, per-group root scale and (optionally) k."""
    ng = -(-cols // 128)
    out = []
    for t in (0, 1):
        q = synth.state_codes(seed, t, 1, 0, rows * cols, fmt, True).reshape(rows, cols)
        k, s, _, _ = synth.state_groups(seed, t, 1, 0, rows * ng)
        k = np.ones(rows * ng, np.float32) if k_one else k
        out.append((q, s.reshape(rows, ng).copy(), k.reshape(rows, ng).copy()))
    return out


def test_forward_hand_case_returns_the_up_codes(orc):
    """gate = 64 everywhere (sigmoid(64) = 1 in double), up with its maximum 448
    in every group, scales 1, k 1: h = 64 up, so without expansion the output
    root scale is 64 and the output codes are the up codes."""
    rows, cols = 3, 256 + 40
    ng = 3
    gq = np.full((rows, cols), 0x68, np.uint8)              # E4M3 0x68 = 2^6
    rng = np.random.default_rng(3)
    mag = rng.integers(1, 0x7F, (rows, cols)).astype(np.uint8)
    mag[:, ::128] = 0x7E
    uq = mag | (rng.integers(0, 2, (rows, cols)).astype(np.uint8) << 7)
    one = np.ones((rows, ng), np.float32)
    oq, os_, ok = orc.swiglu_fp8_forward((gq, one, one), (uq, one, one), E4M3, False)
    assert np.array_equal(oq, uq)
    assert np.all(os_ == 64.0) and np.all(ok == 1.0)
    # with expansion the largest magnitude still maps to 448 and k is in range
    oq, os_, ok = orc.swiglu_fp8_forward((gq, one, one), (uq, one, one), E4M3, True)
    assert np.all((ok >= 1.0) & (ok <= 16.0))
    assert np.all(oq[:, ::128] & 0x7F == 0x7E)


@pytest.mark.parametrize("fmt,expand,k_one", [(E4M3, False, True), (E4M3, True, False),
                                              (E5M2, False, True)])
def test_forward_is_the_composition_of_the_codec_pieces(orc, fmt, expand, k_one):
    rows, cols = 5, 300                                   # a partial last group of 44
    gate, up = _inputs(rows, cols, fmt, 11, k_one)
    got = orc.swiglu_fp8_forward(gate, up, fmt, expand)
    g = orc.group_dequantize(*gate, 1, 128, fmt)
    u = orc.group_dequantize(*up, 1, 128, fmt)
    h = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    want = orc.group_quantize(h.astype(np.float32).astype(np.float64), 1, 128, expand, fmt)
    for a, b in zip(got, want):
        assert np.array_equal(a, b)


def test_backward_hand_case(orc):
    """gate = 64 (sigmoid 1): dgate = dh * up, dup = 64 dh (exact in bf16)."""
    rows, cols = 2, 128
    gq = np.full((rows, cols), 0x68, np.uint8)
    rng = np.random.default_rng(5)
    uq = rng.integers(1, 0x7F, (rows, cols)).astype(np.uint8) | 0x80
    one = np.ones((rows, 1), np.float32)
    dh = synth.grad_bits(3, 0, 1, 0, rows * cols).reshape(rows, cols)
    dg, du = orc.swiglu_fp8_backward(dh, (gq, one, one), (uq, one, one), E4M3)
    u = orc.group_dequantize(uq, one, one, 1, 128, E4M3)
    assert np.array_equal(dg, _bf16_of_f64(_f64_of_bf16(dh) * u))
    assert np.array_equal(du, _bf16_of_f64(64.0 * _f64_of_bf16(dh)))


@pytest.mark.parametrize("fmt,k_one", [(E4M3, True), (E4M3, False), (E5M2, True)])
def test_backward_matches_autograd_on_the_dequantised_inputs(orc, fmt, k_one):
    rows, cols = 4, 300
    gate, up = _inputs(rows, cols, fmt, 12, k_one)
    dh = synth.grad_bits(4, 0, 1, 0, rows * cols).reshape(rows, cols)
    dg, du = orc.swiglu_fp8_backward(dh, gate, up, fmt)
    g = torch.tensor(orc.group_dequantize(*gate, 1, 128, fmt), requires_grad=True)
    u = torch.tensor(orc.group_dequantize(*up, 1, 128, fmt), requires_grad=True)
    (torch.nn.functional.silu(g) * u).backward(torch.from_numpy(_f64_of_bf16(dh)))
    assert np.array_equal(dg, _bf16_of_f64(g.grad.numpy()))
    assert np.array_equal(du, _bf16_of_f64(u.grad.numpy()))
