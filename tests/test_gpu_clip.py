"""Gradient-norm clipping before the step, through the C ABI, against the oracle.

coat_multi_plan_grad_norm: the sum of squares, norm, clip coefficient and
non-finite flag over every gradient of a ragged plan (several tiles per tensor,
ragged tails, empty tensors) against the oracle's double sum; determinism;
Inf/NaN and values whose squares overflow FP32.  coat_adamw_step_multi_clipped:
with a record the test writes (coefficient chosen by the test), against the
oracle step on coef * g; coef = 1 gives the bytes of the plain step; a
found-Inf record leaves every byte alone; and the chain norm -> clipped step
against the oracle's own chain."""
import numpy as np
import pytest
import torch

import fp8_optimizer_state_b200 as coat
import synth
from synth import params as P
from tests.parity import check_master, check_state_all
from tests.test_gpu_adamw import GpuSide, OracleSide, gen_state
from tests.test_gpu_multi import make_sides, plan_of, ragged_sizes

pytestmark = pytest.mark.gpu
H = P.HYPER
HK = {k: H[k] for k in ("lr", "beta1", "beta2", "eps", "wd")}
SUMSQ_RTOL = 1e-6   # FP32 partial sums of 8 exact squares: a few 2^-24 relative


def grads_of(sizes, step, seed=1):
    return [synth.grad_bits(seed, i, step, 0, n) for i, n in enumerate(sizes)]


def load_grads(sides, grads):
    for s, g in zip(sides, grads):
        if g.size:
            s.grad.copy_(torch.from_numpy(g.view(np.int16)))


def oracle_sumsq(orc, grads):
    total, bad = 0.0, False
    for g in grads:
        s, b = orc.grad_sumsq(g)
        total += s
        bad = bad or b
    return total, bad


def test_grad_norm_vs_oracle(orc):
    sizes = ragged_sizes()
    sides = make_sides(sizes, 0, 1)
    grads = grads_of(sizes, 3)
    load_grads(sides, grads)
    plan = plan_of(sides, 0, 1)
    want, bad = oracle_sumsq(orc, grads)
    assert not bad
    norm = np.sqrt(want)
    for max_norm in (norm * 0.25, norm * 4.0, float("inf")):
        buf = coat.new_grad_clip()
        plan.grad_norm(max_norm, buf)
        r = coat.read_grad_clip(buf)
        assert abs(r.sumsq - want) <= SUMSQ_RTOL * want
        assert abs(r.norm - np.float32(norm)) <= 1e-6 * norm
        c_orc = orc.clip_coef(want, np.float32(max_norm))
        # the coefficient follows the sum: within its relative error
        assert abs(r.coef - c_orc) <= 1e-6 * c_orc + 1e-12, (r.coef, c_orc)
        if max_norm > norm:
            assert r.coef == 1.0
        assert r.found_inf == 0 and r.reserved == 0
    # deterministic: same bytes on a second call
    a, b = coat.new_grad_clip(), coat.new_grad_clip()
    plan.grad_norm(1.0, a)
    plan.grad_norm(1.0, b)
    assert torch.equal(a, b)
    plan.destroy()


@pytest.mark.parametrize("n", [1, 7, 8, 9, 7680, 7681, 7680 * 3 + 5])
def test_grad_norm_single_tensor_sizes(orc, n):
    """One tensor of n elements: tails of 1-7 elements, exactly one tile, one
    tile plus one element."""
    side = make_sides([n], 0, 0)[0]
    g = synth.grad_bits(2, 0, 1, 0, n)
    load_grads([side], [g])
    plan = plan_of([side], 0, 0)
    buf = coat.new_grad_clip()
    plan.grad_norm(1.0, buf)
    r = coat.read_grad_clip(buf)
    want, _ = orc.grad_sumsq(g)
    assert abs(r.sumsq - want) <= SUMSQ_RTOL * want
    plan.destroy()


def test_grad_norm_empty_plan():
    sides = make_sides([0, 0], 0, 0)
    plan = plan_of(sides, 0, 0)
    buf = coat.new_grad_clip()
    coat.write_grad_clip(buf, coef=7.0, found_inf=1, sumsq=5.0, norm=3.0)
    plan.grad_norm(2.0, buf)
    r = coat.read_grad_clip(buf)
    assert (r.sumsq, r.norm, r.coef, r.found_inf) == (0.0, 0.0, 1.0, 0)
    plan.destroy()


@pytest.mark.parametrize("bits,finite", [(0x7F80, False), (0xFF80, False), (0x7FC0, False),
                                         (0x7180, True), (0xF27F, True), (0x0001, True)])
def test_grad_norm_special_values(orc, bits, finite):
    """+-Inf and NaN set found_inf; 2^100 and -(2^102 - 2^94) (squares far
    above the FP32 range) and the smallest bf16 subnormal 2^-133 (square far
    below it) are summed as the oracle does."""
    sizes = [3000, 70001, 129]
    sides = make_sides(sizes, 0, 1)
    grads = grads_of(sizes, 2)
    grads[1][12345] = bits
    grads[2][128] = bits
    load_grads(sides, grads)
    plan = plan_of(sides, 0, 1)
    want, bad = oracle_sumsq(orc, grads)
    assert bad == (not finite)
    buf = coat.new_grad_clip()
    plan.grad_norm(1.0, buf)
    r = coat.read_grad_clip(buf)
    assert r.found_inf == (0 if finite else 1)
    if finite:
        assert abs(r.sumsq - want) <= SUMSQ_RTOL * want
        c_orc = orc.clip_coef(want, 1.0)
        assert abs(r.coef - c_orc) <= 1e-6 * c_orc
    else:
        assert not np.isfinite(r.sumsq)
    plan.destroy()


def _identical_sides(orc, sizes, fm, fv, step):
    sides, oras, grads = [], [], []
    for i, n in enumerate(sizes):
        master = synth.master(1, i, 0, n)
        st = gen_state(n, i, step, fm, fv, seed=1)
        sides.append(GpuSide(master, fm, fv).set_state(st))
        oras.append(OracleSide(orc, master, fm, fv).set_state(st))
        grads.append(synth.grad_bits(1, i, step, 0, n))
    load_grads(sides, grads)
    return sides, oras, grads


@pytest.mark.parametrize("fm,fv", [(0, 1), (0, 0), (0, 2)])
@pytest.mark.parametrize("coef", [0.375, 0.0123])
def test_clipped_step_vs_oracle(orc, fm, fv, coef):
    sizes = [5000, 129, 70001, 7680 * 2]
    step = 4
    sides, oras, grads = _identical_sides(orc, sizes, fm, fv, step)
    plan = plan_of(sides, fm, fv)
    buf = coat.new_grad_clip()
    coat.write_grad_clip(buf, coef=coef)
    c = float(np.float32(coef))
    upds = [orc.adamw_step(o.master, o.weight, g, o.mq, o.ms, o.mk, o.vq, o.vs, o.vk, step=step,
                           fmt_m=fm, fmt_v=fv, want_update=True, gscale=c, **HK)
            for o, g in zip(oras, grads)]
    coat.coat_adamw_step_multi_clipped(plan, buf, step=step, **HK)
    coat.coat_check_device_error()
    for n, s, o, u in zip(sizes, sides, oras, upds):
        h = s.host()
        check_master("master", h["master"], o.master, u)
        check_state_all("m", n, fm, h["mq"], h["ms"], h["mk"], o.mq, o.ms, o.mk)
        check_state_all("v", n, fv, h["vq"], h["vs"], h["vk"], o.vq, o.vs, o.vk)
    plan.destroy()


def test_clipped_step_with_coef_one_is_the_plain_step():
    sizes = ragged_sizes()
    a = make_sides(sizes, 0, 1)
    b = make_sides(sizes, 0, 1)
    pa, pb = plan_of(a, 0, 1), plan_of(b, 0, 1)
    buf = coat.new_grad_clip()
    coat.write_grad_clip(buf, coef=1.0)
    for t in (1, 2):
        grads = grads_of(sizes, t)
        load_grads(a, grads)
        load_grads(b, grads)
        coat.coat_adamw_step_multi(pa, step=t, **HK)
        coat.coat_adamw_step_multi_clipped(pb, buf, step=t, **HK)
    coat.coat_check_device_error()
    for sa, sb in zip(a, b):
        ha, hb = sa.host(), sb.host()
        for key in ("master", "weight", "mq", "ms", "mk", "vq", "vs", "vk"):
            assert np.array_equal(ha[key], hb[key]), key
    pa.destroy()
    pb.destroy()


def test_found_inf_leaves_every_byte():
    """A gradient with an Inf: the norm pass flags it and the clipped step
    that follows changes nothing."""
    sizes = [5000, 70001, 129, 0, 7680]
    sides = make_sides(sizes, 0, 1)
    grads = grads_of(sizes, 1)
    grads[1][777] = 0x7F80
    load_grads(sides, grads)
    plan = plan_of(sides, 0, 1)
    before = [s.host() for s in sides]
    buf = coat.new_grad_clip()
    plan.grad_norm(1.0, buf)
    coat.coat_adamw_step_multi_clipped(plan, buf, step=1, **HK)
    coat.coat_check_device_error()
    assert coat.read_grad_clip(buf).found_inf == 1
    for s, h0 in zip(sides, before):
        h1 = s.host()
        for key in ("master", "weight", "mq", "ms", "mk", "vq", "vs", "vk"):
            assert np.array_equal(h0[key], h1[key]), key
    plan.destroy()


def test_norm_then_clipped_step_vs_oracle_chain(orc):
    """Each side runs its own chain: sum of squares, coefficient for a max norm
    a quarter of the norm, step on coef * g."""
    sizes = [5000, 129, 70001, 4096 * 3]
    step = 3
    sides, oras, grads = _identical_sides(orc, sizes, 0, 1, step)
    plan = plan_of(sides, 0, 1)
    want, _ = oracle_sumsq(orc, grads)
    max_norm = float(np.float32(0.25 * np.sqrt(want)))
    c_orc = orc.clip_coef(want, max_norm)
    assert c_orc < 0.3
    upds = [orc.adamw_step(o.master, o.weight, g, o.mq, o.ms, o.mk, o.vq, o.vs, o.vk, step=step,
                           fmt_m=0, fmt_v=1, want_update=True, gscale=c_orc, **HK)
            for o, g in zip(oras, grads)]
    buf = coat.new_grad_clip()
    plan.grad_norm(max_norm, buf)
    coat.coat_adamw_step_multi_clipped(plan, buf, step=step, **HK)
    coat.coat_check_device_error()
    r = coat.read_grad_clip(buf)
    assert abs(r.coef - c_orc) <= 1e-6 * c_orc
    for n, s, o, u in zip(sizes, sides, oras, upds):
        h = s.host()
        check_master("master", h["master"], o.master, u)
        check_state_all("m", n, 0, h["mq"], h["ms"], h["mk"], o.mq, o.ms, o.mk)
        check_state_all("v", n, 1, h["vq"], h["vs"], h["vk"], o.vq, o.vs, o.vk)
    plan.destroy()


def test_clipped_step_replays_from_a_cuda_graph():
    """Norm pass and clipped step enqueue no host round trip, so one training
    step's pair of launches can be captured once and replayed; two replays give
    the bytes of two eager steps."""
    sizes = [5000, 70001, 129, 7680 * 2]
    a = make_sides(sizes, 0, 1)
    b = make_sides(sizes, 0, 1)
    pa, pb = plan_of(a, 0, 1), plan_of(b, 0, 1)
    grads = grads_of(sizes, 1)
    load_grads(a, grads)
    load_grads(b, grads)
    ra, rb = coat.new_grad_clip(), coat.new_grad_clip()
    # eager: two steps on side a (the first call of each entry point also
    # configures its kernels, which a capture must not be the first to do)
    for t in (1, 2):
        pa.grad_norm(0.5, ra)
        coat.coat_adamw_step_multi_clipped(pa, ra, step=t, **HK)
    torch.cuda.synchronize()
    # captured: the same step number both times (the step count is a launch argument)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        pb.grad_norm(0.5, rb)
        coat.coat_adamw_step_multi_clipped(pb, rb, step=1, **HK)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        pb.grad_norm(0.5, rb)
        coat.coat_adamw_step_multi_clipped(pb, rb, step=2, **HK)
    g.replay()
    torch.cuda.synchronize()
    coat.coat_check_device_error()
    for sa, sb in zip(a, b):
        ha, hb = sa.host(), sb.host()
        for key in ("master", "weight", "mq", "ms", "mk", "vq", "vs", "vk"):
            assert np.array_equal(ha[key], hb[key]), key
    assert torch.equal(ra, rb)
    del g
    pa.destroy()
    pb.destroy()
