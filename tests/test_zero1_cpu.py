"""ZeRO-1 data parallelism (coat_zero1_layout and fp8_optimizer_state_b200.zero1)
on the CPU.

The layout is host-only C, so it is checked here directly: over all ranks,
every group of every tensor belongs to exactly one rank, each rank's groups
lie in its own slice of the flat buffer, all shards have one size, the piece
offsets agree with the flat offsets, and every piece's slices pass the
library's own descriptor checks (alignment included) for the step.

The collective plumbing runs with gloo ranks (world sizes 2 and 3).  The
step's kernel needs a GPU, so on the CPU the oracle's step stands in for it
on each rank's pieces (piece_views gives the very slices the kernel would
get); the weights all-gathered afterwards, and every rank's master weights and
FP8 states, must equal the oracle's unsharded step on the summed gradients,
bit for bit, over three steps."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import fp8_optimizer_state_b200 as coat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
G = 128
B = 4 * G          # the layout's block: 4 groups, so per-group floats start 16-byte aligned


def _groups(n):
    return -(-n // G)


def _check_layout(sizes, world):
    owner = {}
    shard = flat = None
    runs = []
    for r in range(world):
        pieces, se, fe, offs = coat.coat_zero1_layout(sizes, world, r)
        assert se % G == 0 and fe == se * world
        assert shard in (None, se) and flat in (None, fe)
        shard, flat = se, fe
        assert offs == list(np.cumsum([0] + [-(-n // B) * B for n in sizes])[:-1])
        assert [p[0] for p in pieces] == sorted(set(p[0] for p in pieces))   # tensor order, one each
        flat_groups = []
        for t, b, n, sb in pieces:
            assert n > 0 and b % B == 0 and sb % B == 0 and b + n <= sizes[t]
            assert b + n == sizes[t] or n % G == 0          # only a tensor's tail is partial
            assert sb + _groups(n) * G <= se
            assert offs[t] + b == r * se + sb                  # the shard is the flat buffer's slice
            for g in range(_groups(n)):
                key = (t, b // G + g)
                assert key not in owner
                owner[key] = r
                flat_groups.append(offs[t] // G + b // G + g)
        # in the rank's slice of the flat buffer, increasing
        assert all(r * se // G <= g < (r + 1) * se // G for g in flat_groups)
        assert flat_groups == sorted(flat_groups)
        runs.append(flat_groups)
    assert sorted(owner) == [(t, g) for t, n in enumerate(sizes) for g in range(_groups(n))]
    total = sum(-(-n // B) for n in sizes)
    assert shard == -(-total // world) * B
    # ranks own consecutive runs in rank order
    nonempty = [x for x in runs if x]
    assert [x[0] for x in nonempty] == sorted(x[0] for x in nonempty)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7, 8, 64])
def test_layout_tiles_every_group_once(world):
    rng = np.random.default_rng(world)
    for sizes in ([300, 128, 1000, 5, 0, 2125], [0], [1], [128] * 9, [4096 * 11008, 4096, 5],
                  list(rng.integers(0, 5000, 40))):
        _check_layout([int(x) for x in sizes], world)


def test_layout_counts_and_errors():
    L = coat.lib()
    import ctypes
    sizes = (ctypes.c_int64 * 3)(300, 0, 257)
    cnt, se, fe = ctypes.c_int(), ctypes.c_int64(), ctypes.c_int64()
    args = (ctypes.byref(cnt), ctypes.byref(se), ctypes.byref(fe), None)
    # counts only
    assert L.coat_zero1_layout(sizes, 3, 128, 2, 0, None, 0, *args) == 1
    assert (cnt.value, se.value, fe.value) == (1, 512, 1024)
    assert L.coat_zero1_layout(sizes, 3, 128, 2, 1, None, 0, *args) == 1
    assert (cnt.value, se.value, fe.value) == (1, 512, 1024)
    pieces = (coat.ShardPiece * 1)()
    assert L.coat_zero1_layout(sizes, 3, 128, 2, 1, pieces, 1, *args) == 0
    assert (pieces[0].tensor, pieces[0].elem_begin, pieces[0].n_elems, pieces[0].shard_begin) == \
        (2, 0, 257, 0)
    bad = [
        (sizes, 0, 128, 2, 0, pieces, 1),    # no tensors
        (sizes, 3, 128, 0, 0, pieces, 1),    # world_size 0
        (sizes, 3, 128, 2, 2, pieces, 1),    # rank out of range
        (sizes, 3, 128, 2, -1, pieces, 1),
        (sizes, 3, 128, 2, 0, None, 1),      # no piece array
        (sizes, 3, 128, 2, 0, pieces, -1),
        (None, 3, 128, 2, 0, pieces, 1),
    ]
    for a in bad:
        assert L.coat_zero1_layout(*a, *args) == 1, a
    assert L.coat_zero1_layout(sizes, 3, 64, 2, 0, pieces, 1, *args) == 3
    neg = (ctypes.c_int64 * 2)(5, -1)
    assert L.coat_zero1_layout(neg, 2, 128, 1, 0, pieces, 1, *args) == 1
    huge = (ctypes.c_int64 * 2)(2 ** 62, 2 ** 62)
    assert L.coat_zero1_layout(huge, 2, 128, 1, 0, pieces, 2, *args) == 1
    # a rank beyond the last group owns nothing
    got, se_, fe_, _ = coat.coat_zero1_layout([100], 4, 3)
    assert got == [] and se_ == 512 and fe_ == 2048


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SIZES = [300, 128, 1000, 5, 0, 2125, 64]
HP = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)
WD_SCALE = [1.0, 0.0, 1.0, 0.5, 1.0, 1.0, 0.0]


def _np(t):
    """A numpy view of a CPU tensor (bf16 as its uint16 patterns)."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _oracle_local_step(z, orc, step, fmt_m, fmt_v, gscale=1.0):
    for piece in z.pieces:
        v = {k: _np(x) for k, x in z.piece_views(piece).items()}
        orc.adamw_step(v["master"], v["weight"], v["grad"], v["m_q"], v["m_scale"], v["m_k"],
                       v["v_q"], v["v_scale"], v["v_k"], step=step, fmt_m=fmt_m, fmt_v=fmt_v,
                       gscale=gscale, **dict(HP, wd=HP["wd"] * WD_SCALE[piece[0]]))


def _plan_status(descs):
    """coat_multi_plan_create's status for host descriptors.  Its checks run
    before any CUDA call, so on a host without a GPU a valid table fails only
    at the device (COAT_ERR_CUDA = 4); a bad one stops at
    COAT_ERR_INVALID_ARG (1) or COAT_ERR_MISALIGNED (2)."""
    import ctypes
    arr = (coat.TensorDesc * len(descs))(*descs)
    h = ctypes.c_void_p()
    return coat.lib().coat_multi_plan_create(ctypes.cast(arr, ctypes.c_void_p), len(descs), G,
                                             0, 0, None, ctypes.byref(h))


def _host_desc(v, shift_scale=0):
    p = {k: x.data_ptr() for k, x in v.items()}
    return coat.TensorDesc(p["master"], p["weight"], p["grad"], p["m_q"],
                           p["m_scale"] + 4 * shift_scale, p["m_k"], p["v_q"], p["v_scale"],
                           p["v_k"], v["master"].numel())


def _check_descriptors(z):
    if not z.pieces:
        return
    views = [z.piece_views(p) for p in z.pieces]
    assert _plan_status([_host_desc(v) for v in views]) == 4
    # the check can fail: one group off is a misaligned scale array
    assert _plan_status([_host_desc(views[0], shift_scale=1)]) == 2


def _setup(rank, world, port, fmt_m, fmt_v, seed):
    """Process group, a Zero1AdamW on the CPU with loaded weights, and the
    unsharded reference state (whole tensors, zero moments)."""
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import synth
    from fp8_optimizer_state_b200.zero1 import Zero1AdamW

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    z = Zero1AdamW(SIZES, device="cpu", fmt_m=fmt_m, fmt_v=fmt_v)
    z.set_wd_scale(WD_SCALE)
    masters = [torch.from_numpy(synth.master(seed, i, 0, n).copy()) for i, n in enumerate(SIZES)]
    z.load_weights(masters)
    ref = []
    for i, n in enumerate(SIZES):
        ng = _groups(n)
        ref.append(dict(master=masters[i].numpy().copy(), weight=np.zeros(n, np.uint16),
                        m_q=np.zeros(ng * G, np.uint8), v_q=np.zeros(ng * G, np.uint8),
                        m_scale=np.ones(ng, np.float32), m_k=np.ones(ng, np.float32),
                        v_scale=np.ones(ng, np.float32), v_k=np.ones(ng, np.float32)))
    return z, ref


def _write_grads(z, rank, seed, step, inf_at=None):
    import synth
    for i, n in enumerate(SIZES):
        bits = synth.grad_bits(seed + rank, i, step, 0, n)
        if inf_at is not None and inf_at[0] == i:
            bits[inf_at[1]] = 0x7F80                      # +Inf in bf16
        z.grad(i).copy_(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16))


def _summed_grads(z):
    """The summed gradients as the reduce-scatter produced them, per tensor."""
    return _summed_grads_of(z, SIZES)


def _reference_step(orc, ref, grads, step, fmt_m, fmt_v, gscale=1.0):
    for i, r in enumerate(ref):
        orc.adamw_step(r["master"], r["weight"], grads[i], r["m_q"], r["m_scale"], r["m_k"],
                       r["v_q"], r["v_scale"], r["v_k"], step=step, fmt_m=fmt_m, fmt_v=fmt_v,
                       gscale=gscale, **dict(HP, wd=HP["wd"] * WD_SCALE[i]))


def _compare(z, ref, tag):
    for i, n in enumerate(SIZES):
        assert np.array_equal(_np(z.weight(i)), ref[i]["weight"]), (tag, i)
    for piece in z.pieces:
        t, b, n, _ = piece
        v = z.piece_views(piece)
        r = ref[t]
        g0, ng = b // G, _groups(n)
        assert np.array_equal(_np(v["master"]).view(np.uint32),
                              r["master"][b:b + n].view(np.uint32)), (tag, t)
        for key in ("m_q", "v_q"):
            assert np.array_equal(_np(v[key])[:n], r[key][b:b + n]), (tag, t, key)
        for key in ("m_scale", "m_k", "v_scale", "v_k"):
            assert np.array_equal(_np(v[key]), r[key][g0:g0 + ng]), (tag, t, key)
    # padding in the flat buffers is never written
    pad = np.ones(z.flat_elems, bool)
    for i, n in enumerate(SIZES):
        pad[z.flat_offsets[i]:z.flat_offsets[i] + n] = False
    assert pad.any() and not _np(z.flat_weight)[pad].any()


def _rank_main(rank, world, port, fmt_m, fmt_v):
    import torch.distributed as dist
    import oracle as orc
    try:
        z, ref = _setup(rank, world, port, fmt_m, fmt_v, 7)
        # the shards are the rank's slices of the flat buffers (in-place collectives)
        lo = 2 * rank * z.shard_elems
        assert z.grad_shard.data_ptr() == z.flat_grad.data_ptr() + lo
        assert z.weight_shard.data_ptr() == z.flat_weight.data_ptr() + lo
        _check_descriptors(z)
        for step in (1, 2, 3):
            _write_grads(z, rank, 20, step)
            if step == 2:            # the asynchronous forms, waited on
                z.reduce_scatter_grads(async_op=True).wait()
            else:
                assert z.reduce_scatter_grads() is None
            _oracle_local_step(z, orc, step, fmt_m, fmt_v)
            if step == 2:
                z.all_gather_weights(async_op=True).wait()
            else:
                z.all_gather_weights()
            _reference_step(orc, ref, _summed_grads(z), step, fmt_m, fmt_v)
            _compare(z, ref, (rank, step))
        dist.barrier()
    finally:
        dist.destroy_process_group()


MAX_NORM = 0.05


def _clip_main(rank, world, port):
    """Clipping over ranks: each rank's sum of squares over its pieces (the
    oracle's, in the norm pass's place), summed by Zero1AdamW's all-reduce;
    the coefficient from that sum must be the one of the whole summed
    gradient, and the clipped states the unsharded clipped step's.  Step 2
    has an Inf in one rank's gradient of a tensor another rank owns: every
    rank must then skip the step."""
    import math
    import torch.distributed as dist
    import oracle as orc
    try:
        z, ref = _setup(rank, world, port, 0, 1, 9)
        coefs = []
        for step in (1, 2, 3):
            _write_grads(z, rank, 40, step, inf_at=(5, 1900) if step == 2 and rank == 0 else None)
            z.reduce_scatter_grads()
            local = sum(orc.grad_sumsq(_np(z.piece_views(p)["grad"]))[0] for p in z.pieces)
            z.clip_sumsq.fill_(local)
            z.allreduce_grad_sumsq()
            total = float(z.clip_sumsq.item())
            grads = _summed_grads(z)
            whole, bad = orc.grad_sumsq(np.concatenate(grads))
            assert bad == (not math.isfinite(total)) == (step == 2)
            if not bad:
                assert abs(total - whole) <= 1e-13 * whole
                coef = orc.clip_coef(total, MAX_NORM)
                assert coef == orc.clip_coef(whole, MAX_NORM)
                coefs.append(coef)
                _oracle_local_step(z, orc, step, 0, 1, gscale=coef)
                _reference_step(orc, ref, grads, step, 0, 1, gscale=coef)
            z.all_gather_weights()
            _compare(z, ref, (rank, step))
        assert all(c < 1.0 for c in coefs)               # the clip was active
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_clipping_over_ranks_equals_the_unsharded_clipped_step(world):
    mp.start_processes(_clip_main, args=(world, _free_port()), nprocs=world, join=True,
                       start_method="spawn")


def _empty_ranks_main(rank, world, port):
    """More ranks than blocks: two blocks over three ranks, so rank 2 owns no
    group (no pieces, no plan) yet takes every collective step; the clipped
    result is the unsharded clipped step's on every rank."""
    import torch.distributed as dist
    import oracle as orc
    import synth
    from fp8_optimizer_state_b200.zero1 import Zero1AdamW

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sizes = [100, 0, 300]
        z = Zero1AdamW(sizes, device="cpu")
        assert (len(z.pieces) > 0) == (rank < 2)
        master = [torch.from_numpy(synth.master(11, i, 0, n).copy()) for i, n in enumerate(sizes)]
        z.load_weights(master)
        ref = [dict(master=m.numpy().copy(), weight=np.zeros(m.numel(), np.uint16),
                    q=[np.zeros(_groups(m.numel()) * G, np.uint8) for _ in range(2)],
                    s=[np.ones(_groups(m.numel()), np.float32) for _ in range(4)])
               for m in master]
        for step in (1, 2):
            grads = []
            for i, n in enumerate(sizes):
                bits = synth.grad_bits(50 + rank, i, step, 0, n)
                z.grad(i).copy_(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16))
            z.reduce_scatter_grads()
            grads = _summed_grads_of(z, sizes)
            local = sum(orc.grad_sumsq(_np(z.piece_views(p)["grad"]))[0] for p in z.pieces)
            if not z.pieces:
                z.clip.zero_()
            z.clip_sumsq.fill_(local)
            z.allreduce_grad_sumsq()
            total = float(z.clip_sumsq.item())
            coef = orc.clip_coef(total, MAX_NORM)
            assert coef == orc.clip_coef(orc.grad_sumsq(np.concatenate(grads))[0], MAX_NORM)
            for piece in z.pieces:
                v = {k: _np(x) for k, x in z.piece_views(piece).items()}
                orc.adamw_step(v["master"], v["weight"], v["grad"], v["m_q"], v["m_scale"],
                               v["m_k"], v["v_q"], v["v_scale"], v["v_k"], step=step, fmt_m=0,
                               fmt_v=0, gscale=coef, **HP)
            z.all_gather_weights()
            for i, r in enumerate(ref):
                orc.adamw_step(r["master"], r["weight"], grads[i], r["q"][0], r["s"][0],
                               r["s"][1], r["q"][1], r["s"][2], r["s"][3], step=step, fmt_m=0,
                               fmt_v=0, gscale=coef, **HP)
                assert np.array_equal(_np(z.weight(i)), r["weight"]), (rank, step, i)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _summed_grads_of(z, sizes):
    import torch.distributed as dist
    full = torch.zeros(z.flat_elems, dtype=torch.bfloat16)
    dist.all_gather_into_tensor(full, z.grad_shard)
    return [_np(full)[o:o + n].copy() for o, n in zip(z.flat_offsets, sizes)]


def test_ranks_without_groups_take_every_collective_step():
    mp.start_processes(_empty_ranks_main, args=(3, _free_port()), nprocs=3, join=True,
                       start_method="spawn")


def _resume_main(rank, world, port, out_dir):
    """Two steps, a checkpoint, a fresh object restored from it: its third
    step gives the same bytes as the original's third step."""
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle as orc
    import synth
    from fp8_optimizer_state_b200.zero1 import Zero1AdamW

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        def run_step(z, step):
            for i, n in enumerate(SIZES):
                bits = synth.grad_bits(30 + rank, i, step, 0, n)
                z.grad(i).copy_(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16))
            z.reduce_scatter_grads()
            _oracle_local_step(z, orc, step, 0, 1)
            z.all_gather_weights()

        a = Zero1AdamW(SIZES, device="cpu", fmt_m=0, fmt_v=1)
        a.set_wd_scale(WD_SCALE)
        a.load_weights([torch.from_numpy(synth.master(8, i, 0, n).copy())
                        for i, n in enumerate(SIZES)])
        run_step(a, 1)
        run_step(a, 2)
        path = os.path.join(out_dir, "rank%d.pt" % rank)
        torch.save(a.state_dict(), path)
        b = Zero1AdamW(SIZES, device="cpu", fmt_m=0, fmt_v=1)
        b.set_wd_scale(WD_SCALE)
        with pytest.raises(ValueError, match="one tensor per size"):
            b.load_weights([torch.zeros(3)])
        b.load_state_dict(torch.load(path))
        assert torch.equal(b.flat_weight.view(torch.int16), a.flat_weight.view(torch.int16))
        run_step(a, 3)
        run_step(b, 3)
        for k in Zero1AdamW._STATE + ("flat_weight",):
            x, y = getattr(a, k), getattr(b, k)
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), k
        # a state saved under another layout is refused
        bad = dict(a.state_dict(), world_size=world + 1)
        with pytest.raises(ValueError, match="another layout"):
            b.load_state_dict(bad)
        bad = dict(a.state_dict(), m_q=a.m_q[:-1].clone())
        with pytest.raises(ValueError, match="m_q"):
            b.load_state_dict(bad)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_checkpoint_resume_is_bit_identical(tmp_path):
    mp.start_processes(_resume_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")


@pytest.mark.parametrize("world,fmt_m,fmt_v", [(2, 0, 0), (3, 0, 1)])
def test_sharded_step_equals_the_unsharded_oracle_step(world, fmt_m, fmt_v):
    mp.start_processes(_rank_main, args=(world, _free_port(), fmt_m, fmt_v), nprocs=world,
                       join=True, start_method="spawn")


def test_local_step_refuses_host_tensors():
    """The product step runs only in the CUDA kernel: on CPU buffers the
    binding refuses to pass host pointers."""
    import torch.distributed as dist
    from fp8_optimizer_state_b200.zero1 import Zero1AdamW
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        z = Zero1AdamW([256], device="cpu")
        with pytest.raises(ValueError, match="CUDA tensor"):
            z.local_step(step=1, **HP)
    finally:
        dist.destroy_process_group()


BF16_U = 2.0 ** -8        # bf16 unit roundoff (8-bit significands, round to nearest)


def _sum_bound_main(rank, world, port):
    """The reduce-scatter sums the ranks' bf16 gradients in bf16 (a reduction
    may round after every addition), so the summed gradient the step receives
    differs from the exact sum.  Any order of world - 1 rounded additions keeps
    |sum - exact| <= (world - 1) u (1 + world u) sum|g_r| (u = 2^-8: each
    partial sum is at most sum|g_r|).  Each rank regenerates every rank's
    gradients, sums its shard exactly in double, and checks the bound on every
    element."""
    import torch.distributed as dist
    import synth
    from fp8_optimizer_state_b200.zero1 import Zero1AdamW
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sizes = [40000, 777, 131072]
        z = Zero1AdamW(sizes, device="cpu")
        worst = 0.0
        for step in (1, 2):
            for i, n in enumerate(sizes):
                bits = synth.grad_bits(50 + rank, i, step, 0, n)
                z.grad(i).copy_(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16))
            z.reduce_scatter_grads()
            got = _np(z.grad_shard).copy()
            for t, b, n, sb in z.pieces:
                parts = [synth.bf16_bits_to_f32(synth.grad_bits(50 + r, t, step, b, n)).astype(np.float64)
                         for r in range(world)]
                exact = np.sum(parts, axis=0)
                mag = np.sum(np.abs(parts), axis=0)
                val = synth.bf16_bits_to_f32(got[sb:sb + n]).astype(np.float64)
                bound = (world - 1) * BF16_U * (1 + world * BF16_U) * mag
                err = np.abs(val - exact)
                assert np.all(err <= bound), (rank, t, float((err - bound).max()))
                nz = mag > 0
                worst = max(worst, float((err[nz] / mag[nz]).max()))
        print("world %d rank %d: worst |sum - exact| / sum|g| = %.3g (bound %.3g)"
              % (world, rank, worst, (world - 1) * BF16_U * (1 + world * BF16_U)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4, 8])
def test_bf16_gradient_sum_is_within_its_rounding_bound(world):
    mp.start_processes(_sum_bound_main, args=(world, _free_port()), nprocs=world, join=True,
                       start_method="spawn")
