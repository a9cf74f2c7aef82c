"""CPU oracle for the COAT FP8-optimizer-state AdamW step, its FP8 codec, the
gradient-clipping pre-step and the FP8 SwiGLU and RMSNorm layers (test
infrastructure).

Plain double-precision C (``coat_oracle.c``) behind a small ctypes loader.
Only the test-suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg import this package; the product library never does.  The
arithmetic, its sources and the readings taken where the COAT pages are
silent are documented at the top of ``coat_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "coat_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

E4M3 = 0
E5M2 = 1
E5M2_FULL = 2   # E5M2 codes, expansion to E5M2's own span

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math",
             "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _P(t):
    return ctypes.POINTER(t)


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.orc_fp8_decode.restype = ctypes.c_double
        L.orc_fp8_decode.argtypes = [ctypes.c_int, ctypes.c_uint]
        L.orc_fp8_encode.restype = ctypes.c_uint
        L.orc_fp8_encode.argtypes = [ctypes.c_int, ctypes.c_float]
        L.orc_fp8_encode_array.restype = None
        L.orc_fp8_encode_array.argtypes = [ctypes.c_int, _P(ctypes.c_float), ctypes.c_int64,
                                           _P(ctypes.c_uint8)]
        L.orc_fmt_max.restype = ctypes.c_double
        L.orc_fmt_max.argtypes = [ctypes.c_int]
        L.orc_target_range.restype = ctypes.c_double
        L.orc_target_range.argtypes = [ctypes.c_int]
        L.orc_float_to_bf16.restype = ctypes.c_uint16
        L.orc_float_to_bf16.argtypes = [ctypes.c_float]
        L.orc_group_params.restype = ctypes.c_double
        L.orc_group_params.argtypes = [_P(ctypes.c_double), ctypes.c_int64, ctypes.c_int,
                                       ctypes.c_int, _P(ctypes.c_float), _P(ctypes.c_float)]
        L.orc_quantize_group.restype = None
        L.orc_quantize_group.argtypes = [_P(ctypes.c_double), ctypes.c_int64, ctypes.c_int,
                                         ctypes.c_int, _P(ctypes.c_uint8), _P(ctypes.c_float),
                                         _P(ctypes.c_float)]
        L.orc_dequant_value.restype = ctypes.c_double
        L.orc_dequant_value.argtypes = [ctypes.c_int, ctypes.c_uint8, ctypes.c_float, ctypes.c_float]
        L.orc_group_quantize.restype = ctypes.c_int
        L.orc_group_quantize.argtypes = [_P(ctypes.c_double), ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, _P(ctypes.c_uint8), ctypes.c_int64,
                                         _P(ctypes.c_float), _P(ctypes.c_float)]
        L.orc_group_dequantize.restype = ctypes.c_int
        L.orc_group_dequantize.argtypes = [_P(ctypes.c_uint8), ctypes.c_int64, _P(ctypes.c_float),
                                           _P(ctypes.c_float), ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           _P(ctypes.c_double), ctypes.c_int64]
        L.orc_adamw_step.restype = ctypes.c_int
        L.orc_adamw_step.argtypes = [_P(ctypes.c_float), _P(ctypes.c_uint16), _P(ctypes.c_uint16),
                                     _P(ctypes.c_uint8), _P(ctypes.c_float), _P(ctypes.c_float),
                                     _P(ctypes.c_uint8), _P(ctypes.c_float), _P(ctypes.c_float),
                                     ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                     ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_int64,
                                     ctypes.c_int, ctypes.c_int, _P(ctypes.c_double)]
        L.orc_adamw_step_scaled.restype = ctypes.c_int
        L.orc_adamw_step_scaled.argtypes = L.orc_adamw_step.argtypes[:-1] + [
            ctypes.c_double, _P(ctypes.c_double)]
        L.orc_grad_sumsq.restype = ctypes.c_double
        L.orc_grad_sumsq.argtypes = [_P(ctypes.c_uint16), ctypes.c_int64, _P(ctypes.c_int)]
        L.orc_clip_coef.restype = ctypes.c_float
        L.orc_clip_coef.argtypes = [ctypes.c_double, ctypes.c_float]
        L.orc_adamw_step_unquantized.restype = ctypes.c_int
        L.orc_adamw_step_unquantized.argtypes = [_P(ctypes.c_double)] * 4 + [
            ctypes.c_int64, ctypes.c_double, ctypes.c_double, ctypes.c_double, ctypes.c_double,
            ctypes.c_double, ctypes.c_int64]
        L.orc_swiglu.restype = ctypes.c_double
        L.orc_swiglu.argtypes = [ctypes.c_double, ctypes.c_double]
        L.orc_swiglu_grad.restype = None
        L.orc_swiglu_grad.argtypes = [ctypes.c_double] * 3 + [_P(ctypes.c_double)] * 2
        _u8, _f, _i = _P(ctypes.c_uint8), _P(ctypes.c_float), ctypes.c_int64
        L.orc_swiglu_fp8_forward.restype = ctypes.c_int
        L.orc_swiglu_fp8_forward.argtypes = [_u8, _i, _f, _f, _i, _u8, _i, _f, _f, _i, _i, _i,
                                             ctypes.c_int, ctypes.c_int, _u8, _i, _f, _f, _i]
        L.orc_swiglu_fp8_backward.restype = ctypes.c_int
        L.orc_swiglu_fp8_backward.argtypes = [_P(ctypes.c_uint16), _i, _u8, _i, _f, _f, _i, _u8,
                                              _i, _f, _f, _i, _i, _i, ctypes.c_int,
                                              _P(ctypes.c_uint16), _i, _P(ctypes.c_uint16), _i]
        L.orc_rmsnorm_fp8_forward.restype = ctypes.c_int
        L.orc_rmsnorm_fp8_forward.argtypes = [_u8, _i, _f, _f, _i, _P(ctypes.c_uint16), _i, _i,
                                              ctypes.c_double, ctypes.c_int, ctypes.c_int, _u8, _i,
                                              _f, _f, _i, _P(ctypes.c_double)]
        L.orc_rmsnorm_fp8_backward.restype = ctypes.c_int
        L.orc_rmsnorm_fp8_backward.argtypes = [_P(ctypes.c_uint16), _i, _u8, _i, _f, _f, _i,
                                               _P(ctypes.c_uint16), _i, _i, ctypes.c_double,
                                               ctypes.c_int, _P(ctypes.c_uint16), _i,
                                               _P(ctypes.c_double)]
        _lib = L
    return _lib


def _ptr(a, ctype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(_P(ctype))


# ----------------------------------------------------------------------------
# FP8 formats
# ----------------------------------------------------------------------------

def fp8_decode(fmt: int, code: int) -> float:
    return lib().orc_fp8_decode(fmt, int(code))


def fp8_decode_table(fmt: int) -> np.ndarray:
    """All 256 code values (float64), from the bit definitions."""
    return np.array([fp8_decode(fmt, c) for c in range(256)], dtype=np.float64)


def fp8_encode(fmt: int, y: float) -> int:
    return int(lib().orc_fp8_encode(fmt, float(y)))


def fp8_encode_array(fmt: int, y) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float32).ravel()
    out = np.zeros(y.size, dtype=np.uint8)
    lib().orc_fp8_encode_array(fmt, _ptr(y, ctypes.c_float), y.size, _ptr(out, ctypes.c_uint8))
    return out


def fmt_max(fmt: int) -> float:
    return lib().orc_fmt_max(fmt)


def target_range(fmt: int = 0) -> float:
    """448 / 2^-9 for E4M3 and E5M2; 57344 / 2^-16 for E5M2_FULL."""
    return lib().orc_target_range(fmt)


def float_to_bf16_bits(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    f = lib().orc_float_to_bf16
    return np.fromiter((f(float(v)) for v in x), dtype=np.uint16, count=x.size)


# ----------------------------------------------------------------------------
# Codec
# ----------------------------------------------------------------------------

def group_params(x, expand: bool, fmt: int):
    """(M, k, s_r) for one group of values."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    k = ctypes.c_float()
    s = ctypes.c_float()
    M = lib().orc_group_params(_ptr(x, ctypes.c_double), x.size, int(bool(expand)), fmt,
                               ctypes.byref(k), ctypes.byref(s))
    return M, k.value, s.value


def quantize_group(x, expand: bool, fmt: int):
    """Codes (uint8), k, s_r for one group."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    codes = np.zeros(x.size, dtype=np.uint8)
    k = ctypes.c_float()
    s = ctypes.c_float()
    lib().orc_quantize_group(_ptr(x, ctypes.c_double), x.size, int(bool(expand)), fmt,
                             _ptr(codes, ctypes.c_uint8), ctypes.byref(k), ctypes.byref(s))
    return codes, k.value, s.value


def dequant_value(fmt: int, code: int, s_r: float, k: float) -> float:
    return lib().orc_dequant_value(fmt, int(code), float(s_r), float(k))


def group_quantize(x, group_rows: int, group_cols: int, expand: bool, fmt: int):
    """x: 2-D array (any float dtype, converted exactly to float64).
    Returns (q uint8 [rows, cols], scale f32 [nbr, nbc], k f32 [nbr, nbc])."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    assert x.ndim == 2
    rows, cols = x.shape
    nbr = -(-rows // group_rows)
    nbc = -(-cols // group_cols)
    q = np.zeros((rows, cols), dtype=np.uint8)
    scale = np.zeros((nbr, nbc), dtype=np.float32)
    k = np.zeros((nbr, nbc), dtype=np.float32)
    rc = lib().orc_group_quantize(_ptr(x, ctypes.c_double), rows, cols, cols, group_rows,
                                  group_cols, int(bool(expand)), fmt, _ptr(q, ctypes.c_uint8),
                                  cols, _ptr(scale, ctypes.c_float), _ptr(k, ctypes.c_float))
    assert rc == 0
    return q, scale, k


def group_dequantize(q, scale, k, group_rows: int, group_cols: int, fmt: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    k = np.ascontiguousarray(k, dtype=np.float32)
    rows, cols = q.shape
    out = np.zeros((rows, cols), dtype=np.float64)
    rc = lib().orc_group_dequantize(_ptr(q, ctypes.c_uint8), cols, _ptr(scale, ctypes.c_float),
                                    _ptr(k, ctypes.c_float), rows, cols, group_rows, group_cols,
                                    fmt, _ptr(out, ctypes.c_double), cols)
    assert rc == 0
    return out


# ----------------------------------------------------------------------------
# AdamW step
# ----------------------------------------------------------------------------

def adamw_step(master, weight_out, grad_bits, m_q, m_scale, m_k, v_q, v_scale, v_k, *, group=128,
               lr, beta1, beta2, eps, wd, step, fmt_m, fmt_v, want_update=False, gscale=1.0):
    """In-place oracle step on numpy arrays (master f32, weight_out u16 or None,
    grad_bits u16, codes u8 padded to whole groups, scale/k f32 per group).
    Returns the per-element |adaptive update| (float64) if want_update."""
    n = master.size
    for a, dt in ((master, np.float32), (grad_bits, np.uint16), (m_q, np.uint8),
                  (v_q, np.uint8), (m_scale, np.float32), (m_k, np.float32),
                  (v_scale, np.float32), (v_k, np.float32)):
        assert a.dtype == dt and a.flags["C_CONTIGUOUS"]
    if weight_out is not None:
        assert weight_out.dtype == np.uint16 and weight_out.size == n
    ng = -(-n // group)
    assert m_q.size >= ng * group and v_q.size >= ng * group and m_k.size >= ng
    upd = np.zeros(n, dtype=np.float64) if want_update else None
    rc = lib().orc_adamw_step_scaled(_ptr(master, ctypes.c_float),
                                     _ptr(weight_out, ctypes.c_uint16),
                                     _ptr(grad_bits, ctypes.c_uint16), _ptr(m_q, ctypes.c_uint8),
                                     _ptr(m_scale, ctypes.c_float), _ptr(m_k, ctypes.c_float),
                                     _ptr(v_q, ctypes.c_uint8), _ptr(v_scale, ctypes.c_float),
                                     _ptr(v_k, ctypes.c_float), n, group, lr, beta1, beta2, eps,
                                     wd, step, fmt_m, fmt_v, float(gscale),
                                     _ptr(upd, ctypes.c_double))
    assert rc == 0
    return upd


def adamw_step_threads(master, weight_out, grad_bits, m_q, m_scale, m_k, v_q, v_scale, v_k, *,
                       threads, group=128, **hyper):
    """adamw_step over `threads` host threads, for timing the oracle on every
    core: the groups are split into contiguous, group-aligned slices and each
    slice is one call of the same C step (ctypes releases the GIL for the
    call).  Groups are independent, so the result is bit for bit that of one
    call over all of them."""
    import concurrent.futures as cf
    n = master.size
    ng = -(-n // group)
    threads = max(1, min(int(threads), ng))
    bounds = [ng * i // threads for i in range(threads + 1)]

    def run(i):
        g0, g1 = bounds[i], bounds[i + 1]
        e0, e1 = g0 * group, min(n, g1 * group)
        if e0 >= e1:
            return
        adamw_step(master[e0:e1], None if weight_out is None else weight_out[e0:e1],
                   grad_bits[e0:e1], m_q[g0 * group:g1 * group], m_scale[g0:g1], m_k[g0:g1],
                   v_q[g0 * group:g1 * group], v_scale[g0:g1], v_k[g0:g1], group=group, **hyper)

    if threads == 1:
        run(0)
        return
    with cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(run, range(threads)))


def grad_sumsq(grad_bits):
    """(sum of squares in double, any non-finite) of bf16 gradient bits."""
    g = np.ascontiguousarray(grad_bits, dtype=np.uint16)
    flag = ctypes.c_int(0)
    s = lib().orc_grad_sumsq(_ptr(g, ctypes.c_uint16), g.size, ctypes.byref(flag))
    return s, bool(flag.value)


def clip_coef(sumsq: float, max_norm: float) -> float:
    return lib().orc_clip_coef(sumsq, max_norm)


def adamw_step_unquantized(p, m, v, g, *, lr, beta1, beta2, eps, wd, step):
    """In-place plain AdamW on float64 arrays."""
    for a in (p, m, v, g):
        assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    rc = lib().orc_adamw_step_unquantized(_ptr(p, ctypes.c_double), _ptr(m, ctypes.c_double),
                                          _ptr(v, ctypes.c_double), _ptr(g, ctypes.c_double),
                                          p.size, lr, beta1, beta2, eps, wd, step)
    assert rc == 0


# ----------------------------------------------------------------------------
# FP8 precision flow through the SwiGLU activation (silu(gate) * up)
# ----------------------------------------------------------------------------

def swiglu(g: float, u: float) -> float:
    return lib().orc_swiglu(float(g), float(u))


def swiglu_grad(g: float, u: float, dh: float):
    """(d/dgate, d/dup) of dh * silu(g) * u."""
    a, b = ctypes.c_double(), ctypes.c_double()
    lib().orc_swiglu_grad(float(g), float(u), float(dh), ctypes.byref(a), ctypes.byref(b))
    return a.value, b.value


def _act(t):
    q, s, k = (np.ascontiguousarray(t[0], dtype=np.uint8), np.ascontiguousarray(t[1], np.float32),
               np.ascontiguousarray(t[2], np.float32))
    assert q.ndim == 2 and s.shape == k.shape and s.shape[0] == q.shape[0]
    assert s.shape[1] == -(-q.shape[1] // 128)
    return q, s, k


def swiglu_fp8_forward(gate, up, fmt: int, expand: bool):
    """gate, up: (codes u8 [rows, cols], scale f32 [rows, ngroups], k f32 [rows, ngroups]).
    Returns the output in the same form, quantised per 1x128 group."""
    gq, gs, gk = _act(gate)
    uq, us, uk = _act(up)
    assert gq.shape == uq.shape
    rows, cols = gq.shape
    ng = gs.shape[1]
    oq = np.zeros((rows, cols), np.uint8)
    os_ = np.zeros((rows, ng), np.float32)
    ok = np.zeros((rows, ng), np.float32)
    u8, f = ctypes.c_uint8, ctypes.c_float
    rc = lib().orc_swiglu_fp8_forward(_ptr(gq, u8), cols, _ptr(gs, f), _ptr(gk, f), ng,
                                      _ptr(uq, u8), cols, _ptr(us, f), _ptr(uk, f), ng, rows, cols,
                                      fmt, int(bool(expand)), _ptr(oq, u8), cols, _ptr(os_, f),
                                      _ptr(ok, f), ng)
    assert rc == 0
    return oq, os_, ok


def swiglu_fp8_backward(dh_bits, gate, up, fmt: int):
    """dh_bits: bf16 bits u16 [rows, cols]; gate / up as for the forward.
    Returns (dgate, dup) as bf16 bits."""
    gq, gs, gk = _act(gate)
    uq, us, uk = _act(up)
    dh = np.ascontiguousarray(dh_bits, dtype=np.uint16)
    assert dh.shape == gq.shape == uq.shape
    rows, cols = gq.shape
    ng = gs.shape[1]
    dg = np.zeros((rows, cols), np.uint16)
    du = np.zeros((rows, cols), np.uint16)
    u8, f, u16 = ctypes.c_uint8, ctypes.c_float, ctypes.c_uint16
    rc = lib().orc_swiglu_fp8_backward(_ptr(dh, u16), cols, _ptr(gq, u8), cols, _ptr(gs, f),
                                       _ptr(gk, f), ng, _ptr(uq, u8), cols, _ptr(us, f),
                                       _ptr(uk, f), ng, rows, cols, fmt, _ptr(dg, u16), cols,
                                       _ptr(du, u16), cols)
    assert rc == 0
    return dg, du


# ----------------------------------------------------------------------------
# FP8 precision flow through RMSNorm (x / sqrt(mean(x^2) + eps) * w)
# ----------------------------------------------------------------------------

def rmsnorm_fp8_forward(x, w_bits, eps, fmt: int, expand: bool, want_rstd=False):
    """x: (codes u8 [rows, d], scale f32 [rows, groups], k f32 [rows, groups]);
    w_bits: bf16 bits u16 [d].  Returns the output (codes, scale, k) [and rstd]."""
    xq, xs, xk = _act(x)
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    rows, d = xq.shape
    assert w.size == d
    ng = xs.shape[1]
    oq = np.zeros((rows, d), np.uint8)
    os_ = np.zeros((rows, ng), np.float32)
    ok = np.zeros((rows, ng), np.float32)
    rstd = np.zeros(rows, np.float64)
    u8, f = ctypes.c_uint8, ctypes.c_float
    rc = lib().orc_rmsnorm_fp8_forward(_ptr(xq, u8), d, _ptr(xs, f), _ptr(xk, f), ng,
                                       _ptr(w, ctypes.c_uint16), rows, d, float(eps), fmt,
                                       int(bool(expand)), _ptr(oq, u8), d, _ptr(os_, f),
                                       _ptr(ok, f), ng, _ptr(rstd, ctypes.c_double))
    assert rc == 0
    return ((oq, os_, ok), rstd) if want_rstd else (oq, os_, ok)


def rmsnorm_fp8_backward(dy_bits, x, w_bits, eps, fmt: int):
    """Returns (dx as bf16 bits u16 [rows, d], dw float64 [d])."""
    xq, xs, xk = _act(x)
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    dy = np.ascontiguousarray(dy_bits, dtype=np.uint16)
    rows, d = xq.shape
    assert dy.shape == (rows, d) and w.size == d
    ng = xs.shape[1]
    dx = np.zeros((rows, d), np.uint16)
    dw = np.zeros(d, np.float64)
    u8, f, u16 = ctypes.c_uint8, ctypes.c_float, ctypes.c_uint16
    rc = lib().orc_rmsnorm_fp8_backward(_ptr(dy, u16), d, _ptr(xq, u8), d, _ptr(xs, f),
                                        _ptr(xk, f), ng, _ptr(w, u16), rows, d, float(eps), fmt,
                                        _ptr(dx, u16), d, _ptr(dw, ctypes.c_double))
    assert rc == 0
    return dx, dw
