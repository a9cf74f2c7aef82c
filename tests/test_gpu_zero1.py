"""ZeRO-1 on one GPU: world size 1 over NCCL runs the product path end to end
(reduce-scatter of the flat gradients, the multi-tensor FP8 step over the
shard's pieces, all-gather of the bf16 weights; with clipping, the norm pass,
an all-reduce of the sum of squares and coat_grad_clip_finalize), which must
give the bits of the plain multi-tensor step on the same tensors.  More ranks need more GPUs;
their partition and collectives are covered by two and three gloo ranks on
the CPU, with the oracle's step in the kernel's place."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import fp8_optimizer_state_b200 as coat
import synth
from synth import params as P

pytestmark = pytest.mark.gpu
H = P.HYPER
G = 128


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _plain_side(master):
    n = master.numel()
    ng = -(-n // G)
    dev = dict(device="cuda")
    return dict(master=master.cuda().clone(), weight=torch.zeros(n, dtype=torch.int16, **dev),
                grad=torch.zeros(n, dtype=torch.int16, **dev),
                m_q=torch.zeros(ng * G, dtype=torch.uint8, **dev),
                v_q=torch.zeros(ng * G, dtype=torch.uint8, **dev),
                m_scale=torch.ones(ng, **dev), m_k=torch.ones(ng, **dev),
                v_scale=torch.ones(ng, **dev), v_k=torch.ones(ng, **dev))


@pytest.mark.parametrize("max_norm", [None, 1e-3])
def test_world_size_one_equals_the_multi_tensor_step(max_norm):
    """max_norm: the clipped step over ranks (norm pass on the shard, an
    all-reduce of the sum of squares, coat_grad_clip_finalize) against the
    plain plan's norm pass and clipped step; the clip records must match too."""
    from fp8_optimizer_state_b200.zero1 import Zero1AdamW
    sizes = [300, 128, 1000, 5, 0, 2125, 4096 * 3 + 7]
    wd_scale = [1.0, 0.0, 1.0, 0.5, 1.0, 1.0, 0.0]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    z = plan = None
    try:
        masters = [torch.from_numpy(synth.master(3, i, 0, n).copy()) for i, n in enumerate(sizes)]
        z = Zero1AdamW(sizes, device="cuda", fmt_m=coat.COAT_E4M3, fmt_v=coat.COAT_E5M2)
        z.set_wd_scale(wd_scale)
        z.load_weights(masters)
        assert [p[0] for p in z.pieces] == [i for i, n in enumerate(sizes) if n]
        sides = [_plain_side(m) for m in masters]
        plan = coat.coat_multi_plan_create(
            [coat.make_desc(s["master"], s["weight"], s["grad"], s["m_q"], s["m_scale"],
                            s["m_k"], s["v_q"], s["v_scale"], s["v_k"]) for s in sides],
            coat.COAT_E4M3, coat.COAT_E5M2)
        plan.set_wd_scale(wd_scale)
        rec = coat.new_grad_clip()
        hp = dict(lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"], eps=H["eps"], wd=H["wd"])
        for t in (1, 2, 3):
            for i, n in enumerate(sizes):
                g = torch.from_numpy(synth.grad_bits(3, i, t, 0, n).view(np.int16)).cuda()
                z.grad(i).view(torch.int16).copy_(g)
                sides[i]["grad"].copy_(g)
            z.step(step=t, max_norm=max_norm, **hp)
            if max_norm is None:
                coat.coat_adamw_step_multi(plan, step=t, **hp)
            else:
                plan.grad_norm(max_norm, rec)
                coat.coat_adamw_step_multi_clipped(plan, rec, step=t, **hp)
                a, b = coat.read_grad_clip(z.clip), coat.read_grad_clip(rec)
                assert bytes(a) == bytes(b), (t, a.sumsq, b.sumsq, a.coef, b.coef)
                assert 0.0 < b.coef < 1.0 and b.found_inf == 0
        coat.coat_check_device_error()
        torch.cuda.synchronize()
        for i, n in enumerate(sizes):
            s = sides[i]
            assert torch.equal(z.weight(i).view(torch.int16), s["weight"]), i
            o, ng = z.flat_offsets[i], -(-n // G)
            assert torch.equal(z.master[o:o + n].view(torch.int32), s["master"].view(torch.int32))
            for key in ("m_q", "v_q"):
                assert torch.equal(getattr(z, key)[o:o + n], s[key][:n]), (i, key)
            for key in ("m_scale", "m_k", "v_scale", "v_k"):
                got = getattr(z, key)[o // G:o // G + ng]
                assert torch.equal(got.view(torch.int32), s[key].view(torch.int32)), (i, key)
        pad = torch.ones(z.flat_elems, dtype=torch.bool, device="cuda")
        for i, n in enumerate(sizes):
            pad[z.flat_offsets[i]:z.flat_offsets[i] + n] = False
        assert not z.flat_weight.view(torch.int16)[pad].any()
    finally:
        if z is not None:
            z.close()
        if plan is not None:
            plan.destroy()
        dist.destroy_process_group()


def test_bench_zero1_mode_line():
    """bench.py --zero1 (one NCCL rank here): the sharded step's JSON line with
    its three phases."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    p = subprocess.run([sys.executable, "bench.py", "--zero1", "--config", "flat-256m", "--steps",
                        "3", "--warmup", "3"], cwd=root, capture_output=True, text=True,
                       timeout=600)
    assert p.returncode == 0, p.stderr[-3000:]
    rec = json.loads([l for l in p.stdout.splitlines() if l.startswith("{")][0])
    assert rec["scaling"] == "strong" and rec["n_gpus"] == 1 and rec["value"] > 0
    assert set(rec["phases_ms"]) == {"reduce_scatter", "step", "all_gather"}
    assert 0 < rec["roofline"]["frac"] < 1.5
