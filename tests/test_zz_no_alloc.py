"""coat_adamw_step_multi_noalloc -- the multi-tensor step for callers that cannot
allocate device memory (for example code running under a framework whose caching
allocator owns all device memory, or a loop that must not allocate after set-up).
Its tensor table lives in a fixed array inside the library instead of a plan's
cudaMalloc'd table.

Checked here through the C ABI: two calls in a row give exactly the bits of the
plan-based entry point on the same inputs, a table of the largest accepted size
gives them too even when the caller overwrites its host table as soon as the
call returns, and a table larger than the fixed array is rejected.  This file is collected last on purpose; it needs nothing
from the other tests and passes on its own in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import fp8_optimizer_state_b200 as coat
import synth
from synth import params as P

pytestmark = pytest.mark.gpu
H = P.HYPER
OK, INVALID, UNSUPPORTED = 0, 1, 3


def make_set(sizes, fm, fv, seed=5):
    """Device buffers for a ragged tensor list, identical for every call with the
    same arguments (generated master and stored state)."""
    out = []
    for i, n in enumerate(sizes):
        ng = -(-n // 128)
        d = dict(master=torch.from_numpy(synth.master(seed, i, 0, n)).cuda(),
                 weight=torch.zeros(n, dtype=torch.int16, device="cuda"),
                 grad=torch.zeros(n, dtype=torch.int16, device="cuda"),
                 mq=torch.zeros(ng * 128, dtype=torch.uint8, device="cuda"),
                 vq=torch.zeros(ng * 128, dtype=torch.uint8, device="cuda"))
        d["mq"][:n] = torch.from_numpy(synth.state_codes(seed, i, 1, 0, n, fm, True)).cuda()
        d["vq"][:n] = torch.from_numpy(synth.state_codes(seed, i, 1, 0, n, fv, False)).cuda()
        km, sm, kv, sv = synth.state_groups(seed, i, 1, 0, ng)
        for key, val in (("mk", km), ("ms", sm), ("vk", kv), ("vs", sv)):
            d[key] = torch.from_numpy(val.copy()).cuda()
        out.append(d)
    return out


def descs_of(tset):
    return [coat.make_desc(d["master"], d["weight"], d["grad"], d["mq"], d["ms"], d["mk"], d["vq"],
                           d["vs"], d["vk"]) for d in tset]


def set_grads(tset, step, seed=5):
    for i, d in enumerate(tset):
        n = d["master"].numel()
        d["grad"].copy_(torch.from_numpy(synth.grad_bits(seed, i, step, 0, n).view(np.int16)))


def test_noalloc_matches_plan_entry_point_on_two_calls():
    fm, fv = 0, 1
    rng = np.random.default_rng(77)
    sizes = list(np.exp(rng.uniform(np.log(1), np.log(200000), 30)).astype(int))
    sizes += [0, 128, 129, 3584, 3585, 3584 * 5, 7]
    a = make_set(sizes, fm, fv)
    b = make_set(sizes, fm, fv)
    plan = coat.coat_multi_plan_create(descs_of(a), fm, fv)
    arr = (coat.TensorDesc * len(sizes))(*descs_of(b))
    stream = torch.cuda.current_stream().cuda_stream
    L = coat.lib()
    for step in (1, 2):
        set_grads(a, step)
        set_grads(b, step)
        coat.coat_adamw_step_multi(plan, step=step, **H)
        st = L.coat_adamw_step_multi_noalloc(ctypes.cast(arr, ctypes.c_void_p), len(sizes), 128,
                                             H["lr"], H["beta1"], H["beta2"], H["eps"], H["wd"],
                                             step, fm, fv, stream)
        assert st == OK
        coat.coat_check_device_error()
        for da, db in zip(a, b):
            for key in ("master", "weight", "mq", "ms", "mk", "vq", "vs", "vk"):
                assert torch.equal(da[key], db[key]), (step, key)
    plan.destroy()


def test_noalloc_rejects_tables_beyond_the_fixed_array():
    L = coat.lib()
    t = make_set([256], 0, 0)[0]
    d = coat.make_desc(t["master"], t["weight"], t["grad"], t["mq"], t["ms"], t["mk"], t["vq"],
                       t["vs"], t["vk"])
    too_many = coat.NOALLOC_MAX_TENSORS + 1
    arr = (coat.TensorDesc * too_many)(*([d] * too_many))
    args = (128, H["lr"], H["beta1"], H["beta2"], H["eps"], H["wd"], 1, 0, 0, None)
    assert L.coat_adamw_step_multi_noalloc(ctypes.cast(arr, ctypes.c_void_p), too_many, *args) == UNSUPPORTED
    assert L.coat_adamw_step_multi_noalloc(ctypes.cast(arr, ctypes.c_void_p), 0, *args) == INVALID
    before = t["master"].clone()
    torch.cuda.synchronize()
    assert torch.equal(t["master"], before)      # nothing was launched


def test_noalloc_full_table_and_host_table_reused_at_once():
    """A table of the largest size (COAT_NOALLOC_MAX_TENSORS tensors, staged in
    chunks) matches the plan-based call, and the host table may be overwritten
    as soon as the call returns: the call has read it by then."""
    fm, fv = 0, 2
    rng = np.random.default_rng(5)
    sizes = [int(x) for x in rng.integers(1, 2500, coat.NOALLOC_MAX_TENSORS)]
    sizes[17] = 0
    a = make_set(sizes, fm, fv, seed=9)
    b = make_set(sizes, fm, fv, seed=9)
    plan = coat.coat_multi_plan_create(descs_of(a), fm, fv)
    stream = torch.cuda.current_stream().cuda_stream
    L = coat.lib()
    for step in (1, 2):
        set_grads(a, step, seed=9)
        set_grads(b, step, seed=9)
        arr = (coat.TensorDesc * len(sizes))(*descs_of(b))
        coat.coat_adamw_step_multi(plan, step=step, **H)
        st = L.coat_adamw_step_multi_noalloc(ctypes.cast(arr, ctypes.c_void_p), len(sizes), 128,
                                             H["lr"], H["beta1"], H["beta2"], H["eps"], H["wd"],
                                             step, fm, fv, stream)
        assert st == OK
        ctypes.memset(arr, 0xFF, ctypes.sizeof(arr))   # the GPU may not have run the copies yet
        coat.coat_check_device_error()
        for da, db in zip(a, b):
            for key in ("master", "weight", "mq", "ms", "mk", "vq", "vs", "vk"):
                assert torch.equal(da[key], db[key]), (step, key)
    plan.destroy()
