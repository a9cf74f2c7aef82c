"""GPU parity of the fused AdamW step (through the C ABI) against the CPU oracle.

Free-running: both sides start from the same seeded inputs (FP32 master, FP32
warm-start moments, bf16 gradients per step), each quantises the warm start with
its own codec and runs its own trajectory; see tests/parity.py for the rules."""
import numpy as np
import pytest
import torch

import fp8_optimizer_state_b200 as coat
import synth
from synth import params as P
from tests.parity import FreeRun, bf16_rne_bits

pytestmark = pytest.mark.gpu
H = P.HYPER
E4M3, E5M2 = 0, 1


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


class GpuSide:
    def __init__(self, master, m0, v0, fmt_m, fmt_v, with_weight=True):
        n = master.size
        ng = -(-n // 128)
        self.n, self.ng, self.fm, self.fv = n, ng, fmt_m, fmt_v
        self.master = to_dev(master)
        self.weight = torch.zeros(n, dtype=torch.int16, device="cuda") if with_weight else None
        self.grad = torch.zeros(n, dtype=torch.int16, device="cuda")
        self.mq = torch.zeros((1, ng * 128), dtype=torch.uint8, device="cuda")
        self.vq = torch.zeros((1, ng * 128), dtype=torch.uint8, device="cuda")
        self.ms, self.mk, self.vs, self.vk = (torch.zeros((1, ng), dtype=torch.float32, device="cuda")
                                              for _ in range(4))
        coat.coat_group_quantize(to_dev(m0).view(1, n), 1, 128, True, fmt_m, self.mq, self.ms, self.mk)
        coat.coat_group_quantize(to_dev(v0).view(1, n), 1, 128, True, fmt_v, self.vq, self.vs, self.vk)

    def step(self, g_bits, t):
        self.grad.copy_(torch.from_numpy(g_bits.view(np.int16)))
        coat.coat_adamw_step(self.master, self.weight, self.grad, self.mq, self.ms, self.mk, self.vq,
                             self.vs, self.vk, lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"],
                             eps=H["eps"], wd=H["wd"], step=t, fmt_m=self.fm, fmt_v=self.fv)

    def host(self):
        torch.cuda.synchronize()
        f = lambda x: x.cpu().numpy().ravel()
        w = None if self.weight is None else self.weight.cpu().numpy().view(np.uint16)
        return dict(master=f(self.master), weight=w, mq=f(self.mq), ms=f(self.ms), mk=f(self.mk),
                    vq=f(self.vq), vs=f(self.vs), vk=f(self.vk))


class OracleSide:
    def __init__(self, orc, master, m0, v0, fmt_m, fmt_v):
        n = master.size
        ng = -(-n // 128)
        self.orc, self.fm, self.fv = orc, fmt_m, fmt_v
        self.master = master.copy()
        self.weight = np.zeros(n, dtype=np.uint16)
        self.mq = np.zeros(ng * 128, np.uint8)
        self.vq = np.zeros(ng * 128, np.uint8)
        q, s, k = orc.group_quantize(m0.reshape(1, n), 1, 128, True, fmt_m)
        self.mq[:n], self.ms, self.mk = q.ravel(), s.ravel().copy(), k.ravel().copy()
        q, s, k = orc.group_quantize(v0.reshape(1, n), 1, 128, True, fmt_v)
        self.vq[:n], self.vs, self.vk = q.ravel(), s.ravel().copy(), k.ravel().copy()

    def step(self, g_bits, t):
        return self.orc.adamw_step(self.master, self.weight, g_bits, self.mq, self.ms, self.mk,
                                   self.vq, self.vs, self.vk, lr=H["lr"], beta1=H["beta1"],
                                   beta2=H["beta2"], eps=H["eps"], wd=H["wd"], step=t,
                                   fmt_m=self.fm, fmt_v=self.fv, want_update=True)


def run_free(orc, n, fmt_m, fmt_v, steps, tensor=0, seed=0):
    master = synth.master(seed, tensor, 0, n)
    m0 = synth.m_warm(seed, tensor, 0, n)
    v0 = synth.v_warm(seed, tensor, 0, n)
    gpu = GpuSide(master, m0, v0, fmt_m, fmt_v)
    ora = OracleSide(orc, master, m0, v0, fmt_m, fmt_v)
    fr = FreeRun(n)
    h = gpu.host()
    fl = fr.check_state("warm m", h["mq"], h["ms"], h["mk"], ora.mq, ora.ms, ora.mk)
    fl |= fr.check_state("warm v", h["vq"], h["vs"], h["vk"], ora.vq, ora.vs, ora.vk)
    fr.exclude(fl)
    for t in range(1, steps + 1):
        g = synth.grad_bits(seed, tensor, t, 0, n)
        gpu.step(g, t)
        upd = ora.step(g, t)
        h = gpu.host()
        fr.check_master("step %d master" % t, h["master"], ora.master, upd)
        assert np.array_equal(h["weight"], bf16_rne_bits(h["master"])), "bf16 copy != RNE(master)"
        same = h["master"] == ora.master
        assert np.array_equal(h["weight"][same & fr.element_mask()],
                              ora.weight[same & fr.element_mask()])
        fl = fr.check_state("step %d m" % t, h["mq"], h["ms"], h["mk"], ora.mq, ora.ms, ora.mk)
        fl |= fr.check_state("step %d v" % t, h["vq"], h["vs"], h["vk"], ora.vq, ora.vs, ora.vk)
        fr.exclude(fl)
    return fr, gpu, ora


def test_tiny_config_free_running_10_steps(orc):
    """Tiny workload: one flat tensor of 1,048,576, E4M3 + E4M3, 10 steps."""
    fr, gpu, ora = run_free(orc, 1 << 20, E4M3, E4M3, 10)
    excluded = int(fr.excluded.sum())
    print("flips per check:", fr.report, "excluded groups:", excluded, "of", fr.ng)
    assert excluded <= 0.05 * fr.ng


@pytest.mark.parametrize("n", [1, 5, 127, 128, 129, 4095, 4096, 4097, 3 * 4096 + 77, 70000])
def test_ragged_sizes_e5m2(orc, n):
    fr, gpu, ora = run_free(orc, n, E4M3, E5M2, 3, tensor=n % 97)
    h = gpu.host()
    ng = -(-n // 128)
    assert not h["mq"][n:].any() and not h["vq"][n:].any()   # padding codes written 0


def test_e5m2_m_and_v(orc):
    run_free(orc, 20000, E5M2, E5M2, 3, tensor=5)


def test_weight_out_optional_and_deterministic():
    n = 50000
    master = synth.master(0, 7, 0, n)
    m0, v0 = synth.m_warm(0, 7, 0, n), synth.v_warm(0, 7, 0, n)
    a = GpuSide(master, m0, v0, E4M3, E5M2, with_weight=True)
    b = GpuSide(master, m0, v0, E4M3, E5M2, with_weight=False)
    for t in (1, 2):
        g = synth.grad_bits(0, 7, t, 0, n)
        a.step(g, t)
        b.step(g, t)
    ha, hb = a.host(), b.host()
    for key in ("master", "mq", "ms", "mk", "vq", "vs", "vk"):
        assert np.array_equal(ha[key], hb[key]), key


def test_resume_from_copied_state_is_bit_identical():
    """Checkpoint/resume: the state is the caller's buffers plus the step count."""
    n = 30000
    master = synth.master(0, 9, 0, n)
    m0, v0 = synth.m_warm(0, 9, 0, n), synth.v_warm(0, 9, 0, n)
    a = GpuSide(master, m0, v0, E4M3, E4M3)
    for t in (1, 2):
        a.step(synth.grad_bits(0, 9, t, 0, n), t)
    saved = {k: getattr(a, k).clone() for k in ("master", "mq", "ms", "mk", "vq", "vs", "vk")}
    b = GpuSide(master, m0, v0, E4M3, E4M3)
    for k, v in saved.items():
        getattr(b, k).copy_(v)
    g3 = synth.grad_bits(0, 9, 3, 0, n)
    a.step(g3, 3)
    b.step(g3, 3)
    ha, hb = a.host(), b.host()
    for key in ("master", "weight", "mq", "ms", "mk", "vq", "vs", "vk"):
        assert np.array_equal(ha[key], hb[key]), key


def test_degenerate_groups_exact(orc):
    """Zero gradient on zero states (k = 1, scale 1, codes 0, pure decay) and
    single-magnitude groups (k = 16, codes +-FMT_MAX)."""
    n = 128 * 6
    master = synth.master(0, 11, 0, n)
    zeros = np.zeros(n, np.float32)
    gpu = GpuSide(master, zeros, zeros, E4M3, E4M3)
    ora = OracleSide(orc, master, zeros, zeros, E4M3, E4M3)
    g = np.zeros(n, dtype=np.float32)
    g[128:256] = 0.25 * np.where(np.arange(128) % 3 == 0, -1, 1)   # one magnitude
    g[256:384] = 2.0 ** -10
    gb = bf16_rne_bits(g)
    for t in (1, 2, 3):
        gpu.step(gb, t)
        ora.step(gb, t)
        h = gpu.host()
        assert np.array_equal(h["mq"], ora.mq) and np.array_equal(h["vq"], ora.vq)
        assert np.array_equal(h["mk"], ora.mk) and np.array_equal(h["vk"], ora.vk)
        assert np.all(h["mk"][[0, 3, 4, 5]] == 1.0) and np.all(h["ms"][[0, 3, 4, 5]] == 1.0)
        assert np.all(h["mk"][[1, 2]] == 16.0)
        assert np.allclose(h["master"], ora.master, rtol=1e-6, atol=1e-10)


def test_zero_length_and_device_error_clear():
    e = torch.empty(0, device="cuda")
    coat.coat_adamw_step(e, None, e, e, e, e, e, e, e, lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8,
                         wd=0.0, step=1)
    coat.coat_check_device_error()
