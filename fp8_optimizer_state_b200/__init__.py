"""Python binding of libcoat.so, the B200 COAT FP8-optimizer-state library.

Argument marshalling only: every function here has the name of a C entry point
in include/coat.h, takes CUDA tensors (or None for optional pointers), passes
their device pointers and the current CUDA stream, and raises CoatError on a
non-OK status.  All arithmetic runs in the library's CUDA kernels; there is no
CPU fallback -- if libcoat.so is missing, every call raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcoat.so")
# the checked build (index checks in every kernel; see include/coat.h)
LIB_CHECKED_PATH = os.path.join(HERE, "libcoat_debug.so")

COAT_E4M3, COAT_E5M2, COAT_E5M2_FULL = 0, 1, 2
COAT_F32, COAT_BF16 = 0, 1
GROUP = 128
STATUS = {0: "COAT_OK", 1: "COAT_ERR_INVALID_ARG", 2: "COAT_ERR_MISALIGNED",
          3: "COAT_ERR_UNSUPPORTED", 4: "COAT_ERR_CUDA", 5: "COAT_ERR_TIMEOUT", 6: "COAT_ERR_NOMEM",
          7: "COAT_ERR_DEVICE_CHECK"}

# (name, restype, argtypes) of every exported entry point
_vp, _i64, _i32, _f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
EXPORTS = [
    ("coat_last_error", ctypes.c_char_p, []),
    ("coat_version", _i32, []),
    ("coat_fp8_encode", _i32, [_vp, _i64, _i32, _vp, _vp]),
    ("coat_fp8_decode", _i32, [_vp, _i64, _i32, _vp, _vp]),
    ("coat_group_quantize", _i32, [_vp, _i32, _i64, _i64, _i64, _i32, _i32, _i32, _i32, _vp, _i64,
                                   _vp, _vp, _vp]),
    ("coat_group_dequantize", _i32, [_vp, _i64, _vp, _vp, _i64, _i64, _i32, _i32, _i32, _vp, _i32,
                                     _i64, _vp]),
    ("coat_adamw_step", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _f32, _f32,
                               _f32, _f32, _f32, _i64, _i32, _i32, _vp]),
    ("coat_multi_plan_create", _i32, [_vp, _i32, _i32, _i32, _i32, _vp, ctypes.POINTER(_vp)]),
    ("coat_adamw_step_multi", _i32, [_vp, _f32, _f32, _f32, _f32, _f32, _i64, _vp]),
    ("coat_multi_plan_destroy", _i32, [_vp]),
    ("coat_multi_plan_set_wd_scale", _i32, [_vp, _vp, _vp]),
    ("coat_multi_plan_info", _i32, [_vp, ctypes.POINTER(_i64), ctypes.POINTER(_i32)]),
    ("coat_check_device_error", _i32, [_vp]),
    ("coat_build_checked", _i32, []),
    ("coat_set_exact_group_params", _i32, [_i32]),
    ("coat_adamw_step_multi_noalloc", _i32, [_vp, _i32, _i32, _f32, _f32, _f32, _f32, _f32, _i64,
                                             _i32, _i32, _vp]),
    ("coat_selftest_wait_timeout", _i32, [_i64, _vp]),
    ("coat_multi_plan_grad_norm", _i32, [_vp, _f32, _vp, _vp]),
    ("coat_adamw_step_multi_clipped", _i32, [_vp, _f32, _f32, _f32, _f32, _f32, _i64, _vp, _vp]),
    ("coat_swiglu_fp8_forward", _i32, [_vp, _vp, _i64, _i64, _i32, _i32, _vp, _vp]),
    ("coat_swiglu_fp8_backward", _i32, [_vp, _i64, _vp, _vp, _i64, _i64, _i32, _vp, _i64, _vp,
                                        _i64, _vp]),
    ("coat_rmsnorm_fp8_forward", _i32, [_vp, _vp, _i64, _i64, _f32, _i32, _i32, _vp, _vp]),
    ("coat_rmsnorm_fp8_workspace_size", _i32, [_i64, ctypes.POINTER(ctypes.c_size_t)]),
    ("coat_rmsnorm_fp8_backward", _i32, [_vp, _i64, _vp, _vp, _i64, _i64, _f32, _i32, _vp, _i64,
                                         _vp, _vp, ctypes.c_size_t, _vp]),
    ("coat_grad_clip_finalize", _i32, [_vp, _f32, _vp]),
    ("coat_zero1_layout", _i32, [_vp, _i32, _i32, _i32, _i32, _vp, _i32, ctypes.POINTER(_i32),
                                 ctypes.POINTER(_i64), ctypes.POINTER(_i64), _vp]),
]
NOALLOC_MAX_TENSORS = 1024


class CoatError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("%s: %s" % (STATUS.get(status, status), message))
        self.status = status


class GradClip(ctypes.Structure):
    """coat_grad_clip (24 bytes; lives in device memory)"""
    _fields_ = [("sumsq", ctypes.c_double), ("norm", _f32), ("coef", _f32),
                ("found_inf", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def new_grad_clip(device=None):
    """A zeroed device buffer holding one coat_grad_clip (a uint8 CUDA tensor)."""
    import torch
    return torch.zeros(ctypes.sizeof(GradClip), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


def read_grad_clip(buf):
    """Copy a coat_grad_clip device buffer to the host (synchronises)."""
    raw = bytes(buf.cpu().numpy().tobytes())
    return GradClip.from_buffer_copy(raw)


def write_grad_clip(buf, coef, found_inf=0, sumsq=0.0, norm=0.0):
    """Fill a coat_grad_clip device buffer from host values."""
    import torch
    rec = GradClip(float(sumsq), float(norm), float(coef), int(found_inf), 0)
    host = torch.frombuffer(bytearray(bytes(rec)), dtype=torch.uint8)
    buf.copy_(host)


class Fp8Act(ctypes.Structure):
    """coat_fp8_act"""
    _fields_ = [("q", _vp), ("scale", _vp), ("k", _vp), ("ldq", _i64), ("lds", _i64)]


def _act(t):
    """(codes [rows, cols] uint8, scale [rows, groups] f32, k [rows, groups] f32) CUDA
    tensors, unit stride along a row (views into a wider buffer are fine)."""
    q, sc, k = t
    if q.dim() != 2 or sc.dim() != 2 or k.dim() != 2 or sc.stride() != k.stride():
        raise ValueError("expected 2-D codes, scale and k with matching strides")
    if q.stride(1) != 1 or sc.stride(1) != 1:
        raise ValueError("rows must be contiguous")
    return Fp8Act(_p(q), _p(sc), _p(k), q.stride(0), sc.stride(0))


def coat_swiglu_fp8_forward(gate, up, fmt, expand_out, out, stream=None):
    """gate, up, out: (codes, scale, k) tensors in the 1x128 layout; out is written."""
    g, u, o = _act(gate), _act(up), _act(out)
    rows, cols = gate[0].shape
    _check(lib().coat_swiglu_fp8_forward(ctypes.byref(g), ctypes.byref(u), rows, cols, fmt,
                                         int(bool(expand_out)), ctypes.byref(o), _s(stream)))


def coat_swiglu_fp8_backward(grad_out, gate, up, fmt, grad_gate, grad_up, stream=None):
    """grad_out, grad_gate, grad_up: bf16 (or int16 bit) [rows, cols] CUDA tensors."""
    g, u = _act(gate), _act(up)
    rows, cols = gate[0].shape
    for t in (grad_out, grad_gate, grad_up):
        if t.dim() != 2 or t.stride(1) != 1 or t.element_size() != 2:
            raise ValueError("expected 2-D bf16 tensors with contiguous rows")
    _check(lib().coat_swiglu_fp8_backward(_p(grad_out), grad_out.stride(0), ctypes.byref(g),
                                          ctypes.byref(u), rows, cols, fmt, _p(grad_gate),
                                          grad_gate.stride(0), _p(grad_up), grad_up.stride(0),
                                          _s(stream)))


def coat_rmsnorm_fp8_forward(x, w, eps, fmt, expand_out, out, stream=None):
    """x, out: (codes, scale, k) tensors in the 1x128 layout; w: bf16 [d] CUDA tensor."""
    xa, oa = _act(x), _act(out)
    rows, d = x[0].shape
    _check(lib().coat_rmsnorm_fp8_forward(ctypes.byref(xa), _p(w), rows, d, eps, fmt,
                                          int(bool(expand_out)), ctypes.byref(oa), _s(stream)))


def coat_rmsnorm_fp8_workspace_size(d):
    n = ctypes.c_size_t()
    _check(lib().coat_rmsnorm_fp8_workspace_size(d, ctypes.byref(n)))
    return n.value


def coat_rmsnorm_fp8_backward(dy, x, w, eps, fmt, dx, dw, workspace, stream=None):
    """dy, dx: bf16 [rows, d]; dw: float32 [d]; workspace: a CUDA buffer of at
    least coat_rmsnorm_fp8_workspace_size(d) bytes."""
    xa = _act(x)
    rows, d = x[0].shape
    for t in (dy, dx):
        if t.dim() != 2 or t.stride(1) != 1 or t.element_size() != 2:
            raise ValueError("expected 2-D bf16 tensors with contiguous rows")
    _check(lib().coat_rmsnorm_fp8_backward(_p(dy), dy.stride(0), ctypes.byref(xa), _p(w), rows, d,
                                           eps, fmt, _p(dx), dx.stride(0), _p(dw), _p(workspace),
                                           workspace.numel() * workspace.element_size(),
                                           _s(stream)))


class TensorDesc(ctypes.Structure):
    """coat_tensor_desc"""
    _fields_ = [("master", _vp), ("weight_bf16_out", _vp), ("grad", _vp), ("m_q", _vp),
                ("m_scale", _vp), ("m_k", _vp), ("v_q", _vp), ("v_scale", _vp), ("v_k", _vp),
                ("n", _i64)]


_lib = None
_loaded = {}


def _load(path):
    if path not in _loaded:
        if not os.path.exists(path):
            raise RuntimeError("%s is not built; run `python -m fp8_optimizer_state_b200.build`"
                               " (add --checked for the checked build)" % path)
        L = ctypes.CDLL(path)
        for name, res, args in EXPORTS:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _loaded[path] = L
    return _loaded[path]


def lib():
    """The loaded library: libcoat.so, or the checked build libcoat_debug.so
    when the environment sets COAT_DEBUG=1 (raises if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_CHECKED_PATH if os.environ.get("COAT_DEBUG") == "1" else LIB_PATH)
    return _lib


@contextlib.contextmanager
def checked_library():
    """Route every call of this module to the checked build inside the block
    (a plan keeps the library that created it)."""
    global _lib
    prev = lib()
    _lib = _load(LIB_CHECKED_PATH)
    try:
        yield _lib
    finally:
        _lib = prev


def _check(status, L=None):
    if status != 0:
        raise CoatError(status, (L or lib()).coat_last_error().decode())


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return t.data_ptr()


def _s(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _dt(t):
    import torch
    if t.dtype == torch.float32:
        return COAT_F32
    if t.dtype in (torch.bfloat16, torch.int16, torch.uint16):
        return COAT_BF16
    raise ValueError("expected float32 or bfloat16 data, got %s" % t.dtype)


def coat_version():
    return lib().coat_version()


def coat_last_error():
    return lib().coat_last_error().decode()


def coat_fp8_encode(y, fmt, q, stream=None):
    """q[i] = FP8 code of FP32 y[i] (nearest, ties to even, saturating)."""
    _check(lib().coat_fp8_encode(_p(y), y.numel(), fmt, _p(q), _s(stream)))


def coat_fp8_decode(q, fmt, out, stream=None):
    _check(lib().coat_fp8_decode(_p(q), q.numel(), fmt, _p(out), _s(stream)))


def coat_group_quantize(x, group_rows, group_cols, expand, fmt, q, scale, k, stream=None):
    """x: 2-D CUDA tensor (f32 or bf16) with unit column stride; q: uint8 [rows, >=cols];
    scale, k: float32 [ceil(rows/gr), ceil(cols/gc)]."""
    rows, cols = x.shape
    _check(lib().coat_group_quantize(_p(x), _dt(x), rows, cols, x.stride(0), group_rows, group_cols,
                                     int(bool(expand)), fmt, _p(q), q.stride(0), _p(scale), _p(k),
                                     _s(stream)))


def coat_group_dequantize(q, scale, k, group_rows, group_cols, fmt, out, stream=None):
    rows, cols = out.shape
    _check(lib().coat_group_dequantize(_p(q), q.stride(0), _p(scale), _p(k), rows, cols, group_rows,
                                       group_cols, fmt, _p(out), _dt(out), out.stride(0),
                                       _s(stream)))


def coat_adamw_step(master, weight_bf16_out, grad, m_q, m_scale, m_k, v_q, v_scale, v_k, *, lr,
                    beta1, beta2, eps, wd, step, fmt_m=COAT_E4M3, fmt_v=COAT_E4M3, group=GROUP,
                    stream=None):
    """One fused AdamW step over FP8 moments (in place); see include/coat.h."""
    _check(lib().coat_adamw_step(_p(master), _p(weight_bf16_out), _p(grad), _p(m_q), _p(m_scale),
                                 _p(m_k), _p(v_q), _p(v_scale), _p(v_k), master.numel(), group, lr,
                                 beta1, beta2, eps, wd, step, fmt_m, fmt_v, _s(stream)))


def make_desc(master, weight_bf16_out, grad, m_q, m_scale, m_k, v_q, v_scale, v_k):
    return TensorDesc(_p(master), _p(weight_bf16_out), _p(grad), _p(m_q), _p(m_scale), _p(m_k),
                      _p(v_q), _p(v_scale), _p(v_k), master.numel())


class coat_multi_plan:
    """Owns a coat_multi_plan_t (created by coat_multi_plan_create)."""

    def __init__(self, handle, descs):
        self.handle = handle
        self._descs = descs
        self._lib = lib()

    def info(self):
        n = ctypes.c_int64()
        c = ctypes.c_int()
        _check(self._lib.coat_multi_plan_info(self.handle, ctypes.byref(n), ctypes.byref(c)),
               self._lib)
        return n.value, c.value

    def set_wd_scale(self, scales, stream=None):
        """Per-tensor weight decay multipliers (coat_multi_plan_set_wd_scale)."""
        arr = (ctypes.c_float * len(scales))(*[float(x) for x in scales])
        _check(self._lib.coat_multi_plan_set_wd_scale(self.handle,
                                                      ctypes.cast(arr, ctypes.c_void_p), _s(stream)),
               self._lib)

    def grad_norm(self, max_norm, clip_buf, stream=None):
        """coat_multi_plan_grad_norm into clip_buf (see new_grad_clip)."""
        coat_multi_plan_grad_norm(self, max_norm, clip_buf, stream)

    def destroy(self):
        if self.handle:
            _check(self._lib.coat_multi_plan_destroy(self.handle), self._lib)
            self.handle = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def coat_multi_plan_create(descs, fmt_m=COAT_E4M3, fmt_v=COAT_E4M3, group=GROUP, stream=None):
    """descs: list of TensorDesc (see make_desc)."""
    arr = (TensorDesc * len(descs))(*descs)
    h = ctypes.c_void_p()
    _check(lib().coat_multi_plan_create(ctypes.cast(arr, ctypes.c_void_p), len(descs), group, fmt_m,
                                        fmt_v, _s(stream), ctypes.byref(h)))
    return coat_multi_plan(h.value, arr)


def coat_adamw_step_multi(plan, *, lr, beta1, beta2, eps, wd, step, stream=None):
    _check(plan._lib.coat_adamw_step_multi(plan.handle, lr, beta1, beta2, eps, wd, step,
                                           _s(stream)), plan._lib)


def coat_multi_plan_grad_norm(plan, max_norm, clip_buf, stream=None):
    if clip_buf.numel() * clip_buf.element_size() < ctypes.sizeof(GradClip):
        raise ValueError("clip_buf must hold %d bytes" % ctypes.sizeof(GradClip))
    _check(plan._lib.coat_multi_plan_grad_norm(plan.handle, max_norm, _p(clip_buf), _s(stream)),
           plan._lib)


def coat_adamw_step_multi_clipped(plan, clip_buf, *, lr, beta1, beta2, eps, wd, step,
                                  stream=None):
    if clip_buf.numel() * clip_buf.element_size() < ctypes.sizeof(GradClip):
        raise ValueError("clip_buf must hold %d bytes" % ctypes.sizeof(GradClip))
    _check(plan._lib.coat_adamw_step_multi_clipped(plan.handle, lr, beta1, beta2, eps, wd, step,
                                                   _p(clip_buf), _s(stream)), plan._lib)


def coat_grad_clip_finalize(clip_buf, max_norm, stream=None):
    """Recompute norm, coef and found_inf of a clip record from its sumsq
    (after the ranks' sums have been added into it)."""
    if clip_buf.numel() * clip_buf.element_size() < ctypes.sizeof(GradClip):
        raise ValueError("clip_buf must hold %d bytes" % ctypes.sizeof(GradClip))
    _check(lib().coat_grad_clip_finalize(_p(clip_buf), max_norm, _s(stream)))


def coat_multi_plan_destroy(plan):
    plan.destroy()


def coat_adamw_step_multi_noalloc(descs, *, lr, beta1, beta2, eps, wd, step, fmt_m=COAT_E4M3,
                                  fmt_v=COAT_E4M3, group=GROUP, stream=None):
    """The multi-tensor step without any allocation (descs: list of TensorDesc,
    at most NOALLOC_MAX_TENSORS).  Reports through the status code only."""
    arr = (TensorDesc * len(descs))(*descs)
    st = lib().coat_adamw_step_multi_noalloc(ctypes.cast(arr, ctypes.c_void_p), len(descs), group,
                                             lr, beta1, beta2, eps, wd, step, fmt_m, fmt_v,
                                             _s(stream))
    if st != 0:
        raise CoatError(st, "coat_adamw_step_multi_noalloc rejected the call")


class ShardPiece(ctypes.Structure):
    """coat_shard_piece"""
    _fields_ = [("tensor", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("elem_begin", _i64), ("n_elems", _i64), ("shard_begin", _i64)]


def coat_zero1_layout(sizes, world_size, rank, group=GROUP):
    """ZeRO-1 partition of tensors of `sizes` elements (host-only; no GPU).
    Returns (pieces, shard_elems, flat_elems, flat_offsets): pieces is this
    rank's list of (tensor, elem_begin, n_elems, shard_begin) tuples."""
    n = len(sizes)
    arr = (_i64 * n)(*[int(x) for x in sizes])
    offs = (_i64 * n)()
    pieces = (ShardPiece * n)()
    cnt, shard, flat = ctypes.c_int(), _i64(), _i64()
    _check(lib().coat_zero1_layout(ctypes.cast(arr, _vp), n, group, world_size, rank,
                                   ctypes.cast(pieces, _vp), n, ctypes.byref(cnt),
                                   ctypes.byref(shard), ctypes.byref(flat),
                                   ctypes.cast(offs, _vp)))
    out = [(p.tensor, p.elem_begin, p.n_elems, p.shard_begin) for p in pieces[:cnt.value]]
    return out, shard.value, flat.value, list(offs)


def coat_set_exact_group_params(on):
    """Group-parameter mode of the step (see include/coat.h); returns the previous one."""
    return lib().coat_set_exact_group_params(int(bool(on)))


@contextlib.contextmanager
def exact_group_params(on=True):
    """Run the block with the step's group-parameter mode set to `on`."""
    prev = coat_set_exact_group_params(on)
    try:
        yield
    finally:
        coat_set_exact_group_params(prev)


def coat_check_device_error(stream=None):
    _check(lib().coat_check_device_error(_s(stream)))


def coat_selftest_wait_timeout(budget_cycles, stream=None):
    """Enqueue one warp whose bounded wait on a barrier nothing arrives on runs
    out; see include/coat.h."""
    _check(lib().coat_selftest_wait_timeout(int(budget_cycles), _s(stream)))
