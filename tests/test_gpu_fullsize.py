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


def test_llama2_7b_full_size_sampled(orc):
    cfg = CONFIGS["llama2-7b"]
    fm, fv = cfg["fmt_m"], cfg["fmt_v"]
    ps = DeviceParamSet(cfg["shapes"](), seed=0)
    try:
        step = 1
        ps.fill_master()
        ps.fill_grad(step)
        ps.fill_states(step, fm, fv)
        descs = []
        for i in range(len(ps)):
            v = ps.views(i)
            descs.append(coat.make_desc(v["master"], v["weight"], v["grad"], v["mq"], v["ms"],
                                        v["mk"], v["vq"], v["vs"], v["vk"]))
        plan = coat.coat_multi_plan_create(descs, fm, fv)
        assert plan.info() == (6738415616, 291)

        rng = np.random.default_rng(50)
        T = len(ps)
        tensors = sorted(set([0, 1, 2, 3, 4, 5, 6, 7, 8, 9, T - 3, T - 2, T - 1]
                             + list(rng.choice(T, 24, replace=False))))
        samples = []
        for i in tensors:
            ng = -(-ps.sizes[i] // 128)
            for gi in sorted(set([0, ng - 1] + list(rng.integers(0, ng, 4)))):
                samples.append((i, int(gi)))

        def grab(i, gi):
            a, cnt, g = ps.group_location(i, gi)
            f = lambda t, lo, hi: t[lo:hi].cpu().numpy()
            return dict(master=f(ps.master, a, a + cnt), weight=f(ps.weight, a, a + cnt).view(np.uint16),
                        mq=f(ps.mq, a, a + 128), vq=f(ps.vq, a, a + 128), ms=f(ps.ms, g, g + 1),
                        mk=f(ps.mk, g, g + 1), vs=f(ps.vs, g, g + 1), vk=f(ps.vk, g, g + 1), cnt=cnt)

        torch.cuda.synchronize()
        coat.coat_adamw_step_multi(plan, step=step,
                                   **{k: H[k] for k in ("lr", "beta1", "beta2", "eps", "wd")})
        coat.coat_check_device_error()
        post = [grab(i, gi) for i, gi in samples]

        flips = 0
        for (i, gi), a in zip(samples, post):
            cnt, e0 = a["cnt"], gi * 128
            # the oracle's inputs, regenerated on the host from the same counters
            master = synth.master(0, i, e0, cnt)
            g = synth.grad_bits(0, i, step, e0, cnt)
            mq = np.zeros(128, np.uint8); vq = np.zeros(128, np.uint8)
            mq[:cnt] = synth.state_codes(0, i, step, e0, cnt, fm, True)
            vq[:cnt] = synth.state_codes(0, i, step, e0, cnt, fv, False)
            km, sm, kv, sv = (x.copy() for x in synth.state_groups(0, i, step, gi, 1))
            ow = np.zeros(cnt, np.uint16)
            upd = orc.adamw_step(master, ow, g, mq, sm, km, vq, sv, kv, step=step, fmt_m=fm,
                                 fmt_v=fv, want_update=True, **H)
            check_master("tensor %d group %d" % (i, gi), a["master"], master, upd)
            assert np.array_equal(a["weight"], bf16_rne_bits(a["master"]))
            flips += check_state_all("m %d/%d" % (i, gi), cnt, fm, a["mq"], a["ms"], a["mk"],
                                     mq, sm, km)[0]
            flips += check_state_all("v %d/%d" % (i, gi), cnt, fv, a["vq"], a["vs"], a["vk"],
                                     vq, sv, kv)[0]
        n_el = 2 * 128 * len(samples)
        print("sampled groups %d, code flips %d of %d codes" % (len(samples), flips, n_el))
        assert flips <= max(2, 1e-4 * n_el)

        # properties over every element
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
