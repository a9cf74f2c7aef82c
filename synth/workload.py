"""Device-resident synthetic parameter sets (PyTorch allocates; the device
generator fills).  Holds no optimizer arithmetic: the warm-start moments are
handed out as FP32 values for the caller to quantise with its own codec.

Layout: one allocation per stream (master f32, grad bf16, weight bf16, m codes,
v codes, and four per-group metadata arrays).  Tensor i starts at element
offset off[i], a multiple of 512, so its groups start at group offset
off[i] / 128, a multiple of 4, and every pointer of the tensor (element and
per-group arrays alike) is 16-byte aligned.
"""
from __future__ import annotations

import numpy as np
import torch

import synth


class DeviceParamSet:
    def __init__(self, shapes, seed=0, with_weight=True, device="cuda"):
        self.names = [s[0] for s in shapes]
        self.sizes = [int(s[1]) for s in shapes]
        self.seed = seed
        padded = [-(-n // 512) * 512 for n in self.sizes]
        self.off = np.concatenate([[0], np.cumsum(padded)]).astype(np.int64)
        total = int(self.off[-1])
        self.total_elements = sum(self.sizes)
        self.total_groups = total // 128
        dev = torch.device(device)
        self.master = torch.empty(total, dtype=torch.float32, device=dev)
        self.grad = torch.empty(total, dtype=torch.int16, device=dev)
        self.weight = torch.empty(total, dtype=torch.int16, device=dev) if with_weight else None
        self.mq = torch.zeros(total, dtype=torch.uint8, device=dev)
        self.vq = torch.zeros(total, dtype=torch.uint8, device=dev)
        g = self.total_groups
        self.ms, self.mk, self.vs, self.vk = (torch.ones(g, dtype=torch.float32, device=dev)
                                              for _ in range(4))

    def __len__(self):
        return len(self.sizes)

    def views(self, i):
        """Per-tensor views: master/grad/weight [n], codes [ceil(n/128)*128],
        metadata [ceil(n/128)]."""
        a, n = int(self.off[i]), self.sizes[i]
        ng = -(-n // 128)
        ga = a // 128
        return dict(master=self.master[a:a + n], grad=self.grad[a:a + n],
                    weight=None if self.weight is None else self.weight[a:a + n],
                    mq=self.mq[a:a + ng * 128], vq=self.vq[a:a + ng * 128],
                    ms=self.ms[ga:ga + ng], mk=self.mk[ga:ga + ng], vs=self.vs[ga:ga + ng],
                    vk=self.vk[ga:ga + ng], n=n, ng=ng)

    def fill_master(self):
        for i in range(len(self)):
            synth.device_master(self.views(i)["master"], self.seed, i)

    def fill_grad(self, step):
        for i in range(len(self)):
            synth.device_grad(self.views(i)["grad"], self.seed, i, step)

    def fill_states(self, step, fmt_m, fmt_v):
        """Stored states (codes, k, root scale) drawn directly by the generator."""
        for i in range(len(self)):
            v = self.views(i)
            n = v["n"]
            if n == 0:
                continue
            synth.device_state_codes(v["mq"][:n], self.seed, i, step, fmt_m, True)
            synth.device_state_codes(v["vq"][:n], self.seed, i, step, fmt_v, False)
            v["mq"][n:].zero_()
            v["vq"][n:].zero_()
            synth.device_state_groups(v["mk"], v["ms"], v["vk"], v["vs"], self.seed, i, step)

    def warm_values(self, i, which, out=None):
        """FP32 warm-start values of moment `which` ('m' or 'v') of tensor i."""
        n = self.sizes[i]
        if out is None or out.numel() < n:
            out = torch.empty(n, dtype=torch.float32, device=self.master.device)
        out = out[:n]
        (synth.device_m_warm if which == "m" else synth.device_v_warm)(out, self.seed, i)
        return out

    def group_location(self, i, gi):
        """(element offset in the flat buffers, valid count, flat group index)."""
        a = int(self.off[i]) + gi * 128
        cnt = min(128, self.sizes[i] - gi * 128)
        return a, cnt, int(self.off[i]) // 128 + gi

    def nbytes(self):
        t = [self.master, self.grad, self.weight, self.mq, self.vq, self.ms, self.mk, self.vs, self.vk]
        return sum(x.numel() * x.element_size() for x in t if x is not None)
