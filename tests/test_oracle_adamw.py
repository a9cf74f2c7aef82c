"""Pins for the oracle's AdamW step over FP8 moments.

The COAT pages name the first and second moments (an Adam-family optimizer,
page "FP8训练新范式：减少40%显存占用，训练速度提高1.4倍", section
"FP8优化器状态") but print no update rule; the problem statement fixes AdamW.
The oracle's AdamW arithmetic is pinned to:
  * a hand-computed single step;
  * the closed form for a constant gradient (m_hat = g, v_hat = g^2 exactly);
  * torch.optim.AdamW in float64 on CPU (a library routine independent of the
    oracle), over several steps with changing gradients;
  * the quantised path reducing to that closed form when every group holds a
    single magnitude (k = 16 and codes +-FMT_MAX dequantise exactly up to the
    FP32 rounding of the stored scale).
"""
import math

import numpy as np
import pytest
import torch

E4M3, E5M2 = 0, 1


def test_hand_step(orc):
    # p=1, g=0.5, m=v=0, t=1, lr=0.1, betas=(0.9, 0.999), eps=1e-8, wd=0.1:
    # m' = 0.05, v' = 2.5e-4, bc1 = 0.1, bc2 = 0.001, sqrt(v')/sqrt(bc2) = 0.5,
    # p = 1*(1-0.01) - 0.1*(0.05/0.1)/(0.5+1e-8) = 0.99 - 0.0999999980 = 0.890000002
    p, m, v, g = (np.array([x], dtype=np.float64) for x in (1.0, 0.0, 0.0, 0.5))
    orc.adamw_step_unquantized(p, m, v, g, lr=0.1, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.1, step=1)
    assert abs(p[0] - (0.99 - 0.05 / 0.50000001)) < 1e-15
    assert abs(p[0] - 0.890000002) < 1e-9
    assert abs(m[0] - 0.05) < 1e-16 and abs(v[0] - 2.5e-4) < 1e-18


@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_constant_gradient_closed_form(orc, wd):
    lr, b1, b2, eps = 1e-3, 0.9, 0.95, 1e-8
    g = np.array([0.5, -0.25, 1e-3, -7.0])
    p0 = np.array([0.3, -0.02, 1.0, 0.0])
    p, m, v = p0.copy(), np.zeros(4), np.zeros(4)
    for t in range(1, 31):
        orc.adamw_step_unquantized(p, m, v, g.copy(), lr=lr, beta1=b1, beta2=b2, eps=eps, wd=wd, step=t)
        d = 1.0 - lr * wd
        closed = d ** t * p0 - lr * g / (np.abs(g) + eps) * sum(d ** i for i in range(t))
        assert np.allclose(p, closed, rtol=1e-12, atol=1e-15)


def test_matches_torch_adamw_float64(orc):
    rng = np.random.default_rng(20)
    n, lr, b1, b2, eps, wd = 1000, 3e-3, 0.9, 0.95, 1e-8, 0.1
    p0 = rng.standard_normal(n) * 0.02
    param = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([param], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd,
                            foreach=False)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t in range(1, 8):
        g = rng.standard_normal(n) * np.exp(rng.uniform(-10, 0, n))
        param.grad = torch.from_numpy(g.copy())
        opt.step()
        orc.adamw_step_unquantized(p, m, v, g, lr=lr, beta1=b1, beta2=b2, eps=eps, wd=wd, step=t)
        st = opt.state[param]
        assert np.allclose(p, param.detach().numpy(), rtol=1e-12, atol=1e-16)
        assert np.allclose(m, st["exp_avg"].numpy(), rtol=1e-12, atol=1e-20)
        assert np.allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-12, atol=1e-24)


def _empty_state(n, group=128):
    ng = -(-n // group)
    z = lambda: np.zeros(ng * group, dtype=np.uint8)
    one = lambda: np.ones(ng, dtype=np.float32)
    return z(), one(), one(), z(), one(), one()


@pytest.mark.parametrize("fmt_v", [E4M3, E5M2])
def test_quantized_step_single_magnitude_groups(orc, fmt_v):
    """Every group holds one gradient magnitude (signs vary), states start at zero:
    each group's m' and v' have one magnitude, so k = 16 and every code is +-FMT_MAX,
    which dequantises back to M up to the FP32 rounding of s_r.  The trajectory must
    then follow the constant-gradient closed form."""
    rng = np.random.default_rng(21)
    n, group = 1000, 128
    lr, b1, b2, eps, wd = 1e-3, 0.9, 0.95, 1e-8, 0.1
    ng = -(-n // group)
    mags = np.float32(2.0) ** rng.integers(-12, 2, ng)   # exact in bf16
    g = np.repeat(mags, group)[:n] * rng.choice([-1.0, 1.0], n)
    g_bits = torch.from_numpy(g.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(g_bits.view(np.int16).astype(np.int32) << 16,
                          g.astype(np.float32).view(np.int32))
    master = (rng.standard_normal(n) * 0.02).astype(np.float32)
    p0 = master.astype(np.float64)
    weight = np.zeros(n, dtype=np.uint16)
    mq, ms, mk, vq, vs, vk = _empty_state(n)
    for t in range(1, 11):
        orc.adamw_step(master, weight, g_bits, mq, ms, mk, vq, vs, vk, lr=lr, beta1=b1, beta2=b2,
                       eps=eps, wd=wd, step=t, fmt_m=E4M3, fmt_v=fmt_v)
        assert np.all(mk == 16.0) and np.all(vk == 16.0)
        # hyperparameters cross the ABI as FP32 and are widened to double
        flr, fwd, feps = (float(np.float32(x)) for x in (lr, wd, eps))
        d = 1.0 - flr * fwd
        closed = d ** t * p0 - flr * g / (np.abs(g) + feps) * sum(d ** i for i in range(t))
        # per step: the FP32 store of p (2^-24 relative) plus ~1e-7 relative on the
        # adaptive part from the FP32 rounding of the stored scales
        tol = 2.0 ** -23 * t * np.abs(closed) + 2e-7 * lr * t
        assert np.all(np.abs(master - closed) <= tol)
        top_m = 0x7E
        top_v = 0x7E if fmt_v == E4M3 else 0x7B
        assert set(np.unique(mq[:n] & 0x7F)) == {top_m}
        assert set(np.unique(vq[:n] & 0x7F)) == {top_v}
        assert not mq[n:].any() and not vq[n:].any()   # padding codes are zero
        ref_bf16 = torch.from_numpy(master).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(weight, ref_bf16)


def test_weight_decay_only(orc):
    """g = 0 and zero moments: the adaptive term is 0/(0+eps) = 0, leaving the
    decoupled decay p (1 - lr wd)^t."""
    n, lr, wd = 300, 1e-2, 0.5
    master = np.linspace(-1, 1, n).astype(np.float32)
    p0 = master.astype(np.float64)
    g = np.zeros(n, dtype=np.uint16)
    mq, ms, mk, vq, vs, vk = _empty_state(n)
    for t in range(1, 6):
        orc.adamw_step(master, None, g, mq, ms, mk, vq, vs, vk, lr=lr, beta1=0.9, beta2=0.95,
                       eps=1e-8, wd=wd, step=t, fmt_m=E4M3, fmt_v=E4M3)
        assert np.allclose(master, p0 * (1 - np.float32(lr) * np.float32(wd)) ** t, rtol=1e-6)
        assert np.all(mk == 1.0) and np.all(ms == 1.0) and not mq.any() and not vq.any()


def test_quantized_close_to_unquantized(orc):
    """With realistic groups (|m| ratio ~1000, v ratio ~10) the FP8-state step stays
    close to the unquantised AdamW step from the same dequantised start."""
    rng = np.random.default_rng(22)
    n, lr, b1, b2, eps, wd = 128 * 40, 1e-4, 0.9, 0.95, 1e-8, 0.1
    sg = np.repeat(10.0 ** rng.uniform(-5, -2, 40), 128)
    m0 = sg * 10.0 ** rng.uniform(-3, 0, n) * rng.choice([-1, 1], n)
    v0 = sg ** 2 * 10.0 ** rng.uniform(-1, 0, n)
    mq = np.zeros(n, np.uint8); vq = np.zeros(n, np.uint8)
    ms = np.zeros(40, np.float32); mk = np.zeros(40, np.float32)
    vs = np.zeros(40, np.float32); vk = np.zeros(40, np.float32)
    for j in range(40):
        sl = slice(128 * j, 128 * (j + 1))
        mq[sl], mk[j], ms[j] = orc.quantize_group(m0[sl], True, E4M3)
        vq[sl], vk[j], vs[j] = orc.quantize_group(v0[sl], True, E4M3)
    m_start = np.array([orc.dequant_value(E4M3, mq[i], ms[i // 128], mk[i // 128]) for i in range(n)])
    v_start = np.array([orc.dequant_value(E4M3, vq[i], vs[i // 128], vk[i // 128]) for i in range(n)])
    master = (rng.standard_normal(n) * 0.02).astype(np.float32)
    p, m, v = master.astype(np.float64), m_start.copy(), v_start.copy()
    for t in range(1, 4):
        g = (sg * rng.standard_normal(n)).astype(np.float32)
        gb = torch.from_numpy(g).to(torch.bfloat16)
        gbits = gb.view(torch.int16).numpy().view(np.uint16)
        orc.adamw_step(master, None, gbits, mq, ms, mk, vq, vs, vk, lr=lr, beta1=b1, beta2=b2,
                       eps=eps, wd=wd, step=t, fmt_m=E4M3, fmt_v=E4M3)
        orc.adamw_step_unquantized(p, m, v, gb.to(torch.float64).numpy(), lr=np.float32(lr),
                                   beta1=np.float32(b1), beta2=np.float32(b2),
                                   eps=np.float32(eps), wd=np.float32(wd), step=t)
    # FP8 moment error (~6% per element at most) moves p by a fraction of lr/bc1 per step
    assert np.max(np.abs(master - p)) < 3 * 0.2 * lr / (1 - b1)
    assert np.median(np.abs(master - p)) < 0.05 * lr / (1 - b1)


# ---------------------------------------------------------------------------
# Gradient-norm clipping and the non-finite check before the step
# ---------------------------------------------------------------------------
def _bf16(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def test_grad_sumsq_closed_forms(orc):
    assert orc.grad_sumsq(_bf16([3.0, 4.0])) == (25.0, False)          # a 3-4-5 triangle
    assert orc.grad_sumsq(_bf16([0.5] * 1000)) == (250.0, False)
    assert orc.grad_sumsq(_bf16([-2.0 ** -10] * 64)) == (64 * 2.0 ** -20, False)
    assert orc.grad_sumsq(np.zeros(0, np.uint16)) == (0.0, False)
    for bad in (float("inf"), float("-inf"), float("nan")):
        assert orc.grad_sumsq(_bf16([1.0, bad, 2.0]))[1] is True


def test_grad_sumsq_matches_numpy_on_random_bf16(orc):
    """The sum of squares of 100,000 bf16 values against numpy's float64 dot
    product (a library routine; squares of bf16 values are exact in double)."""
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)       # truncation: any bf16 will do
    vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    s, bad = orc.grad_sumsq(bits)
    assert not bad
    assert abs(s - float(np.dot(vals, vals))) <= 1e-12 * s


def test_clip_coef_closed_forms(orc):
    # norm 5: max_norm / (norm + 1e-6), rounded to FP32, when below 1
    assert orc.clip_coef(25.0, 1.0) == np.float32(1.0 / (5.0 + 1e-6))
    assert orc.clip_coef(25.0, 2.5) == np.float32(2.5 / (5.0 + 1e-6))
    assert orc.clip_coef(25.0, 10.0) == 1.0          # already below the limit
    assert orc.clip_coef(0.0, 1.0) == 1.0            # zero gradient
    assert orc.clip_coef(25.0, float("inf")) == 1.0  # no limit


def test_scaled_step_is_the_step_on_the_scaled_gradient(orc):
    """gscale = 0.5 gives exactly the state of the plain step on bf16 gradients
    halved exactly (every value here is far from the bf16 subnormal range)."""
    n = 128 * 5 + 17
    rng = np.random.default_rng(3)
    g = rng.normal(0, 1e-3, n).astype(np.float32)
    g[np.abs(g) < 1e-6] = 1e-6
    gb = _bf16(g)
    gh = _bf16(torch.from_numpy(gb.view(np.int16)).view(torch.bfloat16).float().numpy() * 0.5)
    m0 = np.random.default_rng(4).normal(0, 0.02, n).astype(np.float32)
    res = []
    for bits, gs in ((gb, 0.5), (gh, 1.0)):
        master = m0.copy()
        ng = -(-n // 128)
        st = [np.zeros(ng * 128, np.uint8), np.ones(ng, np.float32), np.ones(ng, np.float32),
              np.zeros(ng * 128, np.uint8), np.ones(ng, np.float32), np.ones(ng, np.float32)]
        for t in (1, 2):
            orc.adamw_step(master, None, bits, st[0], st[1], st[2], st[3], st[4], st[5], lr=1e-3,
                           beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1, step=t, fmt_m=E4M3,
                           fmt_v=E4M3, gscale=gs)
        res.append((master, st))
    (ma, sa), (mb, sb) = res
    assert np.array_equal(ma, mb)
    for x, y in zip(sa, sb):
        assert np.array_equal(x, y)


def test_threaded_timing_form_is_bit_identical(orc):
    """The all-cores timing helper (group-aligned slices, one C call each, on
    host threads) gives exactly the bytes of one call over every group."""
    import synth
    n, fm, fv = 100_003, E4M3, E5M2
    ng = -(-n // 128)
    master = synth.master(0, 3, 0, n)
    g = synth.grad_bits(0, 3, 2, 0, n)
    mq = np.zeros(ng * 128, np.uint8)
    vq = np.zeros(ng * 128, np.uint8)
    mq[:n] = synth.state_codes(0, 3, 2, 0, n, fm, True)
    vq[:n] = synth.state_codes(0, 3, 2, 0, n, fv, False)
    km, sm, kv, sv = synth.state_groups(0, 3, 2, 0, ng)
    hyper = dict(lr=1e-4, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1, step=2, fmt_m=fm, fmt_v=fv)
    outs = []
    for threads in (None, 7):
        st = [a.copy() for a in (master, mq, sm, km, vq, sv, kv)]
        w = np.zeros(n, np.uint16)
        if threads is None:
            orc.adamw_step(st[0], w, g, st[1], st[2], st[3], st[4], st[5], st[6], **hyper)
        else:
            orc.adamw_step_threads(st[0], w, g, st[1], st[2], st[3], st[4], st[5], st[6],
                                   threads=threads, **hyper)
        outs.append(st + [w])
    for a, b in zip(*outs):
        assert np.array_equal(a, b)
