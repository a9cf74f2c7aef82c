"""Full-size parity: the Llama-2-7B-shaped parameter list (6.74e9 parameters,
68 GB resident) in the launch configuration the benchmark times (one
multi-tensor launch per step).  The oracle checks sampled groups one by one
(its inputs regenerated on the host from the same counters); properties that
hold at any size are checked over every element on the device."""
import numpy as np
import pytest
import torch

import fp8_optimizer_state_b200 as coat
import synth
from synth.params import CONFIGS, HYPER as H
from synth.workload import DeviceParamSet
from tests.parity import bf16_rne_bits, check_master, check_state_all

pytestmark = pytest.mark.gpu


def _build(fm, fv, step, config="llama2-7b"):
    cfg = CONFIGS[config]
    ps = DeviceParamSet(cfg["shapes"](), seed=0)
    ps.fill_master()
    ps.fill_grad(step)
    ps.fill_states(step, fm, fv)
    return ps


def _desc(ps, i):
    v = ps.views(i)
    return coat.make_desc(v["master"], v["weight"], v["grad"], v["mq"], v["ms"], v["mk"], v["vq"],
                          v["vs"], v["vk"])


def _samples(ps, seed):
    rng = np.random.default_rng(seed)
    T = len(ps)
    tensors = sorted(set([0, 1, 2, 3, 4, 5, 6, 7, 8, 9, T - 3, T - 2, T - 1]
                         + list(rng.choice(T, 24, replace=False))))
    samples = []
    for i in tensors:
        ng = -(-ps.sizes[i] // 128)
        for gi in sorted(set([0, ng - 1] + list(rng.integers(0, ng, 4)))):
            samples.append((i, int(gi)))
    return samples


def _grab(ps, i, gi):
    a, cnt, g = ps.group_location(i, gi)
    f = lambda t, lo, hi: t[lo:hi].cpu().numpy()
    return dict(master=f(ps.master, a, a + cnt), weight=f(ps.weight, a, a + cnt).view(np.uint16),
                mq=f(ps.mq, a, a + 128), vq=f(ps.vq, a, a + 128), ms=f(ps.ms, g, g + 1),
                mk=f(ps.mk, g, g + 1), vs=f(ps.vs, g, g + 1), vk=f(ps.vk, g, g + 1), cnt=cnt)


def _check_samples(orc, samples, post, step, fm, fv, gscale=1.0, same_out=None):
    """The oracle on each sampled group, its inputs regenerated on the host from
    the same counters; returns the number of code flips.  same_out (a list):
    receives, per sampled group and moment, whether k and the root scale equal
    the oracle's bit for bit."""
    flips = 0
    for (i, gi), a in zip(samples, post):
        cnt, e0 = a["cnt"], gi * 128
        master = synth.master(0, i, e0, cnt)
        g = synth.grad_bits(0, i, step, e0, cnt)
        mq = np.zeros(128, np.uint8); vq = np.zeros(128, np.uint8)
        mq[:cnt] = synth.state_codes(0, i, step, e0, cnt, fm, True)
        vq[:cnt] = synth.state_codes(0, i, step, e0, cnt, fv, False)
        km, sm, kv, sv = (x.copy() for x in synth.state_groups(0, i, step, gi, 1))
        ow = np.zeros(cnt, np.uint16)
        upd = orc.adamw_step(master, ow, g, mq, sm, km, vq, sv, kv, step=step, fmt_m=fm,
                             fmt_v=fv, want_update=True, gscale=gscale, **H)
        check_master("tensor %d group %d" % (i, gi), a["master"], master, upd)
        assert np.array_equal(a["weight"], bf16_rne_bits(a["master"]))
        flips += check_state_all("m %d/%d" % (i, gi), cnt, fm, a["mq"], a["ms"], a["mk"],
                                 mq, sm, km)[0]
        flips += check_state_all("v %d/%d" % (i, gi), cnt, fv, a["vq"], a["vs"], a["vk"],
                                 vq, sv, kv)[0]
        if same_out is not None:
            same_out.append(bool(a["mk"][0] == km[0] and a["ms"][0] == sm[0]))
            same_out.append(bool(a["vk"][0] == kv[0] and a["vs"][0] == sv[0]))
    n_el = 2 * 128 * len(samples)
    print("sampled groups %d, code flips %d of %d codes" % (len(samples), flips, n_el))
    assert flips <= max(2, 1e-4 * n_el)
    return flips


def test_llama2_7b_full_size_sampled(orc):
    cfg = CONFIGS["llama2-7b"]
    fm, fv = cfg["fmt_m"], cfg["fmt_v"]
    step = 1
    ps = _build(fm, fv, step)
    try:
        plan = coat.coat_multi_plan_create([_desc(ps, i) for i in range(len(ps))], fm, fv)
        assert plan.info() == (6738415616, 291)
        samples = _samples(ps, 50)
        torch.cuda.synchronize()
        coat.coat_adamw_step_multi(plan, step=step,
                                   **{k: H[k] for k in ("lr", "beta1", "beta2", "eps", "wd")})
        coat.coat_check_device_error()
        post = [_grab(ps, i, gi) for i, gi in samples]
        _check_samples(orc, samples, post, step, fm, fv)

        # properties over every element
        T = len(ps)
        for i in range(T):
            v = ps.views(i)
            assert torch.equal(v["weight"], v["master"].to(torch.bfloat16).view(torch.int16)), i
            assert bool(torch.isfinite(v["master"]).all())
        for k in (ps.mk, ps.vk):
            assert bool(((k >= 1) & (k <= 16)).all())
        for s_ in (ps.ms, ps.vs):
            assert bool((torch.isfinite(s_) & (s_ > 0)).all())
        plan.destroy()
    finally:
        del ps
        torch.cuda.empty_cache()


def test_llama2_7b_full_size_sampled_exact_group_params(orc):
    """The full-size launch with exact group parameters: besides the tolerances,
    k and the root scale of the sampled groups are the oracle's bits (the
    correctly rounded values of the definition), except where an FP32 near-tie
    hides the true extreme."""
    cfg = CONFIGS["llama2-7b"]
    fm, fv = cfg["fmt_m"], cfg["fmt_v"]
    step = 3
    ps = _build(fm, fv, step)
    try:
        plan = coat.coat_multi_plan_create([_desc(ps, i) for i in range(len(ps))], fm, fv)
        samples = _samples(ps, 51)
        torch.cuda.synchronize()
        with coat.exact_group_params(True):
            coat.coat_adamw_step_multi(plan, step=step,
                                       **{k: H[k] for k in ("lr", "beta1", "beta2", "eps", "wd")})
        coat.coat_check_device_error()
        post = [_grab(ps, i, gi) for i, gi in samples]
        same = []
        _check_samples(orc, samples, post, step, fm, fv, same_out=same)
        print("k and scale bit-identical: %d of %d sampled group moments" % (sum(same), len(same)))
        assert sum(same) >= 0.99 * len(same)
        plan.destroy()
    finally:
        del ps
        torch.cuda.empty_cache()


def test_llama2_7b_grad_norm_and_clipped_step_full_size(orc):
    """The gradient-norm pass over all 6.74e9 gradients in one launch: the
    oracle's sum on every tensor of up to 2^24 elements that a sample picks
    (each through its own one-tensor plan), the whole-list sum against the sum
    of all 291 one-tensor sums (the same FP32 partials, so only the double
    summation order differs); then the clipped step with a coefficient the
    test writes, sampled against the oracle step on coef * g."""
    cfg = CONFIGS["llama2-7b"]
    fm, fv = cfg["fmt_m"], cfg["fmt_v"]
    step = 2
    ps = _build(fm, fv, step)
    try:
        T = len(ps)
        plan = coat.coat_multi_plan_create([_desc(ps, i) for i in range(T)], fm, fv)
        whole = coat.new_grad_clip()
        plan.grad_norm(1.0, whole)
        rw = coat.read_grad_clip(whole)
        assert rw.found_inf == 0 and np.isfinite(rw.sumsq) and rw.sumsq > 0

        rng = np.random.default_rng(51)
        small = [i for i in range(T) if ps.sizes[i] <= (1 << 24)]
        picked = set(rng.choice(small, 4, replace=False)) | {small[0], small[-1]}
        per = []
        buf = coat.new_grad_clip()
        for i in range(T):
            p1 = coat.coat_multi_plan_create([_desc(ps, i)], fm, fv)
            p1.grad_norm(1.0, buf)
            r = coat.read_grad_clip(buf)
            per.append(r.sumsq)
            if i in picked:
                want, bad = orc.grad_sumsq(synth.grad_bits(0, i, step, 0, ps.sizes[i]))
                assert not bad
                assert abs(r.sumsq - want) <= 1e-6 * want, (i, r.sumsq, want)
            p1.destroy()
        total = float(np.sum(np.array(per, dtype=np.float64)))
        assert abs(rw.sumsq - total) <= 1e-9 * total
        assert rw.norm == np.float32(np.sqrt(rw.sumsq))

        coef = 0.375
        coat.write_grad_clip(whole, coef=coef)
        samples = _samples(ps, 52)
        torch.cuda.synchronize()
        coat.coat_adamw_step_multi_clipped(plan, whole, step=step,
                                           **{k: H[k] for k in ("lr", "beta1", "beta2", "eps",
                                                                "wd")})
        coat.coat_check_device_error()
        post = [_grab(ps, i, gi) for i, gi in samples]
        _check_samples(orc, samples, post, step, fm, fv, gscale=coef)
        plan.destroy()
    finally:
        del ps
        torch.cuda.empty_cache()


def test_llama2_13b_full_size_sampled(orc):
    """The 13B-shaped list (363 tensors, 1.30e10 parameters, E4M3 m and v; about
    132 GB resident) in one multi-tensor launch, sampled groups against the
    oracle and the per-element properties."""
    cfg = CONFIGS["llama2-13b"]
    fm, fv = cfg["fmt_m"], cfg["fmt_v"]
    step = 1
    ps = _build(fm, fv, step, "llama2-13b")
    try:
        plan = coat.coat_multi_plan_create([_desc(ps, i) for i in range(len(ps))], fm, fv)
        assert plan.info() == (13015864320, 363)
        samples = _samples(ps, 53)
        torch.cuda.synchronize()
        coat.coat_adamw_step_multi(plan, step=step,
                                   **{k: H[k] for k in ("lr", "beta1", "beta2", "eps", "wd")})
        coat.coat_check_device_error()
        post = [_grab(ps, i, gi) for i, gi in samples]
        _check_samples(orc, samples, post, step, fm, fv)
        for k in (ps.mk, ps.vk):
            assert bool(((k >= 1) & (k <= 16)).all())
        for s_ in (ps.ms, ps.vs):
            assert bool((torch.isfinite(s_) & (s_ > 0)).all())
        for i in range(len(ps)):      # per tensor: a whole-array temporary would not fit
            assert bool(torch.isfinite(ps.views(i)["master"]).all()), i
        plan.destroy()
    finally:
        del ps
        torch.cuda.empty_cache()
