"""Multi-tensor launcher: one launch over a ragged tensor list must give exactly
the bits of per-tensor coat_adamw_step calls, and match the oracle."""
import numpy as np
import pytest
import torch

import fp8_optimizer_state_b200 as coat
import synth
from synth import params as P
from tests.parity import check_master, check_state_all
from tests.test_gpu_adamw import GpuSide, OracleSide, gen_state

pytestmark = pytest.mark.gpu
H = P.HYPER


def ragged_sizes():
    rng = np.random.default_rng(40)
    sizes = list(np.exp(rng.uniform(np.log(1), np.log(300000), 40)).astype(int))
    return sizes + [1, 127, 128, 129, 4096, 4097, 8192 * 3, 0, 5]


def make_sides(sizes, fm, fv):
    sides = []
    for i, n in enumerate(sizes):
        master = synth.master(1, i, 0, n)
        sides.append(GpuSide(master, fm, fv).warm_start(synth.m_warm(1, i, 0, n),
                                                        synth.v_warm(1, i, 0, n)))
    return sides


def plan_of(sides, fm, fv):
    descs = [coat.make_desc(s.master, s.weight, s.grad, s.mq, s.ms, s.mk, s.vq, s.vs, s.vk)
             for s in sides]
    return coat.coat_multi_plan_create(descs, fm, fv)


@pytest.mark.parametrize("fm,fv", [(0, 1), (0, 0)])
def test_multi_equals_single_calls(fm, fv):
    sizes = ragged_sizes()
    a = make_sides(sizes, fm, fv)
    b = make_sides(sizes, fm, fv)
    plan = plan_of(b, fm, fv)
    assert plan.info() == (sum(sizes), len(sizes))
    for t in (1, 2, 3):
        for i, (sa, sb) in enumerate(zip(a, b)):
            g = synth.grad_bits(1, i, t, 0, sizes[i])
            sb.grad.copy_(torch.from_numpy(g.view(np.int16)))
            sa.step(g, t)
        coat.coat_adamw_step_multi(plan, lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"],
                                   eps=H["eps"], wd=H["wd"], step=t)
    coat.coat_check_device_error()
    for sa, sb in zip(a, b):
        ha, hb = sa.host(), sb.host()
        for key in ("master", "weight", "mq", "ms", "mk", "vq", "vs", "vk"):
            assert np.array_equal(ha[key], hb[key]), key
    plan.destroy()


def test_multi_vs_oracle(orc):
    """One multi-tensor launch from identical generated states matches the oracle."""
    sizes = [5000, 129, 70001, 4096 * 3]
    sides, oras = [], []
    for i, n in enumerate(sizes):
        master = synth.master(1, i, 0, n)
        st = gen_state(n, i, 4, 0, 1, seed=1)
        sides.append(GpuSide(master, 0, 1).set_state(st))
        oras.append(OracleSide(orc, master, 0, 1).set_state(st))
    plan = plan_of(sides, 0, 1)
    upds = []
    for i, (s, o) in enumerate(zip(sides, oras)):
        g = synth.grad_bits(1, i, 4, 0, sizes[i])
        s.grad.copy_(torch.from_numpy(g.view(np.int16)))
        upds.append(o.step(g, 4))
    coat.coat_adamw_step_multi(plan, lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"],
                               eps=H["eps"], wd=H["wd"], step=4)
    coat.coat_check_device_error()
    for n, s, o, u in zip(sizes, sides, oras, upds):
        h = s.host()
        check_master("master", h["master"], o.master, u)
        check_state_all("m", n, 0, h["mq"], h["ms"], h["mk"], o.mq, o.ms, o.mk)
        check_state_all("v", n, 1, h["vq"], h["vs"], h["vk"], o.vq, o.vs, o.vk)
    plan.destroy()


def test_per_tensor_weight_decay():
    """wd_scale 1 / 0 per tensor gives exactly the bits of single calls with wd
    and with wd = 0 (e.g. normalisation weights excluded from decay); a scale of
    0.5 matches the oracle with half the decay."""
    sizes = [4096 + 3, 700, 128 * 40, 333]
    scales = [1.0, 0.0, 1.0, 0.0]
    a = make_sides(sizes, 0, 1)
    b = make_sides(sizes, 0, 1)
    plan = plan_of(b, 0, 1)
    plan.set_wd_scale(scales)
    for t in (1, 2):
        for i, (sa, sb) in enumerate(zip(a, b)):
            g = synth.grad_bits(1, i, t, 0, sizes[i])
            sb.grad.copy_(torch.from_numpy(g.view(np.int16)))
            sa.grad.copy_(torch.from_numpy(g.view(np.int16)))
            coat.coat_adamw_step(sa.master, sa.weight, sa.grad, sa.mq, sa.ms, sa.mk, sa.vq, sa.vs,
                                 sa.vk, lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"],
                                 eps=H["eps"], wd=H["wd"] * scales[i], step=t, fmt_m=0, fmt_v=1)
        coat.coat_adamw_step_multi(plan, lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"],
                                   eps=H["eps"], wd=H["wd"], step=t)
    coat.coat_check_device_error()
    for sa, sb in zip(a, b):
        ha, hb = sa.host(), sb.host()
        for key in ("master", "weight", "mq", "ms", "mk", "vq", "vs", "vk"):
            assert np.array_equal(ha[key], hb[key]), key
    plan.destroy()


def test_half_weight_decay_vs_oracle(orc):
    n = 70001
    master = synth.master(1, 9, 0, n)
    st = gen_state(n, 9, 3, 0, 1, seed=1)
    side = GpuSide(master, 0, 1).set_state(st)
    ora = OracleSide(orc, master, 0, 1).set_state(st)
    plan = plan_of([side], 0, 1)
    plan.set_wd_scale([0.5])
    g = synth.grad_bits(1, 9, 3, 0, n)
    side.grad.copy_(torch.from_numpy(g.view(np.int16)))
    upd = orc.adamw_step(ora.master, ora.weight, g, ora.mq, ora.ms, ora.mk, ora.vq, ora.vs,
                         ora.vk, lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"], eps=H["eps"],
                         wd=H["wd"] * 0.5, step=3, fmt_m=0, fmt_v=1, want_update=True)
    coat.coat_adamw_step_multi(plan, lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"],
                               eps=H["eps"], wd=H["wd"], step=3)
    coat.coat_check_device_error()
    h = side.host()
    check_master("master", h["master"], ora.master, upd)
    check_state_all("m", n, 0, h["mq"], h["ms"], h["mk"], ora.mq, ora.ms, ora.mk)
    check_state_all("v", n, 1, h["vq"], h["vs"], h["vk"], ora.vq, ora.vs, ora.vk)
    with pytest.raises(coat.CoatError):
        plan.set_wd_scale([-1.0])
    plan.destroy()
