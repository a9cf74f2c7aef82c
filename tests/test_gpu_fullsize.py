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
from tests.parity import rel_err, compare_codes, K_RTOL, SCALE_RTOL, MASTER_RTOL, bf16_rne_bits

pytestmark = pytest.mark.gpu


def test_llama2_7b_full_size_sampled(orc):
    cfg = CONFIGS["llama2-7b"]
    fm, fv = cfg["fmt_m"], cfg["fmt_v"]
    ps = DeviceParamSet(cfg["shapes"](), seed=0)
    try:
        ps.fill_master()
        ps.fill_grad(1)
        tmp = None
        for i in range(len(ps)):
            v = ps.views(i)
            tmp = ps.warm_values(i, "m", tmp)
            coat.coat_group_quantize(tmp.view(1, -1), 1, 128, True, fm, v["mq"].view(1, -1),
                                     v["ms"].view(1, -1), v["mk"].view(1, -1))
            tmp = ps.warm_values(i, "v", tmp)
            coat.coat_group_quantize(tmp.view(1, -1), 1, 128, True, fv, v["vq"].view(1, -1),
                                     v["vs"].view(1, -1), v["vk"].view(1, -1))
        del tmp
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
        pre = [grab(i, gi) for i, gi in samples]
        coat.coat_adamw_step_multi(plan, step=1, **{k: H[k] for k in ("lr", "beta1", "beta2", "eps", "wd")})
        coat.coat_check_device_error()
        post = [grab(i, gi) for i, gi in samples]

        warm_flips = step_flips = compared = 0
        for (i, gi), b, a in zip(samples, pre, post):
            cnt, e0 = b["cnt"], gi * 128
            master = synth.master(0, i, e0, cnt)
            assert np.array_equal(b["master"], master)       # device generator == host generator
            m0, v0 = synth.m_warm(0, i, e0, cnt), synth.v_warm(0, i, e0, cnt)
            g = synth.grad_bits(0, i, 1, e0, cnt)
            mq = np.zeros(128, np.uint8); vq = np.zeros(128, np.uint8)
            mq[:cnt], mk, ms = orc.quantize_group(m0, True, fm)
            vq[:cnt], vk, vs = orc.quantize_group(v0, True, fv)
            ms, mk, vs, vk = (np.array([x], np.float32) for x in (ms, mk, vs, vk))
            assert rel_err(b["mk"], mk).max() <= K_RTOL and rel_err(b["vk"], vk).max() <= K_RTOL
            assert rel_err(b["ms"], ms).max() <= SCALE_RTOL and rel_err(b["vs"], vs).max() <= SCALE_RTOL
            d1, x1 = compare_codes(b["mq"], mq)
            d2, x2 = compare_codes(b["vq"], vq)
            assert x1 <= 1 and x2 <= 1
            if d1.any() or d2.any():
                warm_flips += int(d1.sum() + d2.sum())
                continue
            om = master.copy()
            ow = np.zeros(cnt, np.uint16)
            upd = orc.adamw_step(om, ow, g, mq, ms, mk, vq, vs, vk, step=1, fmt_m=fm, fmt_v=fv,
                                 want_update=True, **H)
            tol = MASTER_RTOL * (np.abs(om.astype(np.float64)) + upd)
            assert np.all(np.abs(a["master"].astype(np.float64) - om) <= tol), (i, gi)
            assert np.array_equal(a["weight"], bf16_rne_bits(a["master"]))
            assert rel_err(a["mk"], mk).max() <= K_RTOL and rel_err(a["vk"], vk).max() <= K_RTOL
            assert rel_err(a["ms"], ms).max() <= SCALE_RTOL and rel_err(a["vs"], vs).max() <= SCALE_RTOL
            d1, x1 = compare_codes(a["mq"], mq)
            d2, x2 = compare_codes(a["vq"], vq)
            assert x1 <= 1 and x2 <= 1
            step_flips += int(d1.sum() + d2.sum())
            compared += 1
        n_el = 2 * 128 * len(samples)
        print("sampled groups %d, compared %d, warm-start flips %d, step flips %d"
              % (len(samples), compared, warm_flips, step_flips))
        assert compared >= 0.9 * len(samples)
        assert warm_flips + step_flips <= max(4, 1e-4 * n_el * 2)

        # properties over every element
        for i in range(T):
            v = ps.views(i)
            assert torch.equal(v["weight"], v["master"].to(torch.bfloat16).view(torch.int16)), i
            assert bool(torch.isfinite(v["master"]).all())
        for k in (ps.mk, ps.vk):
            assert bool(((k >= 1) & (k <= 16)).all())
        for s in (ps.ms, ps.vs):
            assert bool((torch.isfinite(s) & (s > 0)).all())
        plan.destroy()
    finally:
        del ps
        torch.cuda.empty_cache()
