"""Guard bytes and the checked build: the library's stand-ins for a device
memory checker.

Every buffer a call reads or writes is the middle of a larger allocation whose
head and tail (256 bytes each) hold a fixed byte pattern, the tail starting
right at the buffer's last byte; after the call both must be intact, so a
kernel that wrote one element past either end of any buffer would be caught.
Each case runs twice on the same generated inputs: with the release library
(libcoat.so) and with the checked build (libcoat_debug.so), whose kernels check
every index they derive before the access and count failures on the device.
The checked run must report no failed check (coat_check_device_error), and
both runs must give the same bytes.  Sizes are ragged on purpose: 1, 127, 129,
4097 elements, a tile plus one, partial 1x128 groups and 128x128 blocks, the
narrowest layer widths."""
import ctypes

import numpy as np
import pytest
import torch

import fp8_optimizer_state_b200 as coat
import synth
from synth import params as P

pytestmark = pytest.mark.gpu
H = P.HYPER
GUARD = 256
PATTERN = 0xA5
TILE = 7680   # elements of the step kernel's tile


class Arena:
    """Buffers carved out of guarded allocations."""

    def __init__(self):
        self.blocks = []

    def alloc(self, shape, dtype, fill=None):
        shape = (shape,) if isinstance(shape, int) else tuple(shape)
        n = int(np.prod(shape))
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        blk = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.blocks.append(blk)
        view = blk[GUARD:GUARD + nbytes].view(dtype).view(shape)
        if fill is not None:
            view.copy_(torch.as_tensor(np.ascontiguousarray(fill)).view(dtype).view(shape))
        return view

    def check(self, tag):
        torch.cuda.synchronize()
        for i, blk in enumerate(self.blocks):
            head, tail = blk[:GUARD], blk[-GUARD:]
            assert bool((head == PATTERN).all()), "%s: buffer %d: bytes before it were written" % (tag, i)
            assert bool((tail == PATTERN).all()), "%s: buffer %d: bytes after it were written" % (tag, i)


def both(run):
    """run() with the release library and with the checked build; returns both
    results after the guard and device-error checks."""
    out = []
    for checked in (False, True):
        if checked:
            with coat.checked_library() as L:
                assert L.coat_build_checked() == 1
                out.append(run("checked"))
                coat.coat_check_device_error()   # no index check failed
        else:
            assert coat.lib().coat_build_checked() == 0
            out.append(run("release"))
            coat.coat_check_device_error()
    return out


def same(a, b, tag):
    assert len(a) == len(b)
    for i, (x, y) in enumerate(zip(a, b)):
        assert np.array_equal(x, y), "%s: output %d differs between the builds" % (tag, i)


def host(*ts):
    torch.cuda.synchronize()
    return [t.detach().cpu().contiguous().view(torch.uint8).numpy().copy() for t in ts]


STEP_SIZES = [1, 127, 128, 129, 4097, TILE + 1, 3 * TILE + 77]


def step_buffers(A, n, fm, fv, tensor):
    ng = -(-n // 128)
    mq = np.zeros(ng * 128, np.uint8)
    vq = np.zeros(ng * 128, np.uint8)
    mq[:n] = synth.state_codes(0, tensor, 1, 0, n, fm, True)
    vq[:n] = synth.state_codes(0, tensor, 1, 0, n, fv, False)
    km, sm, kv, sv = synth.state_groups(0, tensor, 1, 0, ng)
    return dict(master=A.alloc(n, torch.float32, synth.master(0, tensor, 0, n)),
                weight=A.alloc(n, torch.int16),
                grad=A.alloc(n, torch.int16, synth.grad_bits(0, tensor, 1, 0, n).view(np.int16)),
                mq=A.alloc(ng * 128, torch.uint8, mq), ms=A.alloc(ng, torch.float32, sm),
                mk=A.alloc(ng, torch.float32, km), vq=A.alloc(ng * 128, torch.uint8, vq),
                vs=A.alloc(ng, torch.float32, sv), vk=A.alloc(ng, torch.float32, kv))


KEYS = ("master", "weight", "mq", "ms", "mk", "vq", "vs", "vk")


@pytest.mark.parametrize("n", STEP_SIZES)
def test_single_tensor_step(n):
    fm, fv = 0, 1

    def run(tag):
        A = Arena()
        b = step_buffers(A, n, fm, fv, n % 31)
        for t in (1, 2):
            coat.coat_adamw_step(b["master"], b["weight"], b["grad"], b["mq"], b["ms"], b["mk"],
                                 b["vq"], b["vs"], b["vk"], step=t, fmt_m=fm, fmt_v=fv, **H)
        A.check("step n=%d %s" % (n, tag))
        return host(*(b[k] for k in KEYS))

    rel, chk = both(run)
    same(rel, chk, "step n=%d" % n)


def test_multi_tensor_step_norm_and_clipped_step():
    sizes = STEP_SIZES + [0, 300]
    fm, fv = 0, 2

    def run(tag):
        A = Arena()
        bufs = [step_buffers(A, n, fm, fv, i) if n else None for i, n in enumerate(sizes)]
        descs = []
        for b in bufs:
            if b is None:
                descs.append(coat.TensorDesc(None, None, None, None, None, None, None, None, None, 0))
            else:
                descs.append(coat.make_desc(b["master"], b["weight"], b["grad"], b["mq"], b["ms"],
                                            b["mk"], b["vq"], b["vs"], b["vk"]))
        plan = coat.coat_multi_plan_create(descs, fm, fv)
        clip = A.alloc(ctypes.sizeof(coat.GradClip), torch.uint8, np.zeros(24, np.uint8))
        coat.coat_adamw_step_multi(plan, step=1, **H)
        plan.grad_norm(1e-3, clip)
        coat.coat_adamw_step_multi_clipped(plan, clip, step=2, **H)
        plan.destroy()
        A.check("multi %s" % tag)
        return host(clip, *(b[k] for b in bufs if b is not None for k in KEYS))

    rel, chk = both(run)
    same(rel, chk, "multi")


def test_noalloc_step():
    sizes = [1, 129, 4097, TILE + 1]

    def run(tag):
        A = Arena()
        bufs = [step_buffers(A, n, 0, 1, i) for i, n in enumerate(sizes)]
        descs = [coat.make_desc(b["master"], b["weight"], b["grad"], b["mq"], b["ms"], b["mk"],
                                b["vq"], b["vs"], b["vk"]) for b in bufs]
        coat.coat_adamw_step_multi_noalloc(descs, step=1, fmt_m=0, fmt_v=1, **H)
        A.check("noalloc %s" % tag)
        return host(*(b[k] for b in bufs for k in KEYS))

    rel, chk = both(run)
    same(rel, chk, "noalloc")


CODEC_SHAPES = [(1, 1), (3, 127), (129, 129), (5, 4097), (130, 300)]


@pytest.mark.parametrize("rows,cols", CODEC_SHAPES)
@pytest.mark.parametrize("gr", [1, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_codec_quantize_dequantize(rows, cols, gr, dtype):
    """Row strides are the ABI's (multiples of 16 bytes), so the last row of a
    buffer ends in the tail guard and earlier rows are followed by padding."""
    nbr, nbc = -(-rows // gr), -(-cols // 128)
    bits = synth.activations_bits(0, rows + cols, 0, rows * cols).view(np.int16)
    xf = synth.bf16_bits_to_f32(bits.view(np.uint16)).reshape(rows, cols)

    def strided(A, dt, fill=None):
        per16 = 16 // torch.empty(0, dtype=dt).element_size()
        ld = -(-cols // per16) * per16
        full = A.alloc((rows - 1) * ld + cols, dt)
        view = full.as_strided((rows, cols), (ld, 1))
        if fill is not None:
            view.copy_(torch.as_tensor(np.ascontiguousarray(fill)).view(dt).cuda())
        return view

    def run(tag):
        A = Arena()
        if dtype == torch.bfloat16:
            x = strided(A, torch.int16, bits.reshape(rows, cols)).view(torch.bfloat16)
        else:
            x = strided(A, torch.float32, xf)
        outs = []
        for expand in (0, 1):
            q = strided(A, torch.uint8)
            s = A.alloc((nbr, nbc), torch.float32)
            k = A.alloc((nbr, nbc), torch.float32)
            coat.coat_group_quantize(x, gr, 128, expand, 0, q, s, k)
            ob = strided(A, torch.int16).view(torch.bfloat16)
            of = strided(A, torch.float32)
            coat.coat_group_dequantize(q, s, k, gr, 128, 0, ob)
            coat.coat_group_dequantize(q, s, k, gr, 128, 0, of)
            outs += [q, s, k, ob, of]
        A.check("codec %dx%d gr=%d %s %s" % (rows, cols, gr, dtype, tag))
        return host(*outs)

    rel, chk = both(run)
    same(rel, chk, "codec %dx%d" % (rows, cols))


def fp8_input(A, rows, cols, seed):
    ng = -(-cols // 128)
    q = synth.state_codes(seed, 7, 1, 0, rows * cols, 0, True).reshape(rows, cols)
    s = np.full((rows, ng), 0.25, np.float32)
    k = np.ones((rows, ng), np.float32)
    return (A.alloc((rows, cols), torch.uint8, q), A.alloc((rows, ng), torch.float32, s),
            A.alloc((rows, ng), torch.float32, k))


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 144), (2, 4112)])
def test_swiglu_layer(rows, cols):
    ng = -(-cols // 128)

    def run(tag):
        A = Arena()
        gate, up = fp8_input(A, rows, cols, 1), fp8_input(A, rows, cols, 2)
        out = (A.alloc((rows, cols), torch.uint8), A.alloc((rows, ng), torch.float32),
               A.alloc((rows, ng), torch.float32))
        coat.coat_swiglu_fp8_forward(gate, up, 0, True, out)
        dh = A.alloc((rows, cols), torch.int16,
                     synth.grad_bits(0, 3, 1, 0, rows * cols).view(np.int16).reshape(rows, cols))
        dg = A.alloc((rows, cols), torch.int16)
        du = A.alloc((rows, cols), torch.int16)
        coat.coat_swiglu_fp8_backward(dh, gate, up, 0, dg, du)
        A.check("swiglu %dx%d %s" % (rows, cols, tag))
        return host(*out, dg, du)

    rel, chk = both(run)
    same(rel, chk, "swiglu %dx%d" % (rows, cols))


@pytest.mark.parametrize("rows,d", [(1, 128), (5, 384)])
def test_rmsnorm_layer(rows, d):
    ng = d // 128

    def run(tag):
        A = Arena()
        x = fp8_input(A, rows, d, 3)
        w = A.alloc(d, torch.int16, (synth.f32_to_bf16_bits(
            1.0 + 0.1 * np.sin(np.arange(d, dtype=np.float32)))).view(np.int16))
        out = (A.alloc((rows, d), torch.uint8), A.alloc((rows, ng), torch.float32),
               A.alloc((rows, ng), torch.float32))
        coat.coat_rmsnorm_fp8_forward(x, w, 1e-6, 0, False, out)
        dy = A.alloc((rows, d), torch.int16,
                     synth.grad_bits(0, 4, 1, 0, rows * d).view(np.int16).reshape(rows, d))
        dx = A.alloc((rows, d), torch.int16)
        dw = A.alloc(d, torch.float32)
        ws = A.alloc(coat.coat_rmsnorm_fp8_workspace_size(d), torch.uint8)
        coat.coat_rmsnorm_fp8_backward(dy, x, w, 1e-6, 0, dx, dw, ws)
        A.check("rmsnorm %dx%d %s" % (rows, d, tag))
        return host(*out, dx, dw)

    rel, chk = both(run)
    same(rel, chk, "rmsnorm %dx%d" % (rows, d))
