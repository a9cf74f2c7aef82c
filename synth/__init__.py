"""Seeded synthetic inputs for the COAT FP8-state AdamW step.

This module holds none of the method's arithmetic: it only turns counters into
numbers.  Both the CPU oracle's tests and the GPU path draw their inputs from
here, so the two sides see the same bits.  There are two implementations of one
generator: NumPy on the host (this file) and CUDA on the device
(``csrc/synth.cu``).  They agree bit for bit because every step is an integer
operation or a single correctly rounded IEEE operation (no library
transcendental is used anywhere).

Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
as easy as 1, 2, 3", SC'11): 10 rounds of two 32x32->64 multiplies with
multipliers 0xD2511F53 and 0xCD9E8D57, a word permutation, and a Weyl key
schedule with increments 0x9E3779B9 and 0xBB67AE85.  Key = (seed, stream id),
counter = (element index lo, element index hi, tensor id, step).

Value recipes (the workload descriptions give the distributions):
  * normal: Irwin-Hall sum of the four 32-bit words, centred and scaled to unit
    variance in double: z = (u0+u1+u2+u3 - (2^33-2)) * sqrt(3) / 2^32.  It stands
    in for N(0,1) (|z| <= 3.47).
  * log-uniform on [lo, hi]: a uniform draw over the FP32 bit patterns between lo
    and hi (equal mass per octave, linear within an octave).
  * master ~ 0.02 z; per-group gradient scale s_g log-uniform on [1e-5, 1e-2];
    grad = bf16(s_g z) redrawn per step; warm-start |m| log-uniform on
    [1e-3 s_g, s_g] with a random sign (max/min ~ 1000), v log-uniform on
    [0.1 s_g^2, s_g^2] (max/min ~ 10); activations z with 0.1% of entries x100;
    weight matrices 0.02 z.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

# stream ids (Philox key word 1)
MASTER, GRAD, MSTATE, VSTATE, GSCALE, ACT, ACT_OUTLIER, WEIGHT = 1, 2, 3, 4, 5, 6, 7, 8
MCODE, VCODE, GSTATE = 9, 10, 11

_PHILOX_M0 = np.uint64(0xD2511F53)
_PHILOX_M1 = np.uint64(0xCD9E8D57)
_PHILOX_W0 = np.uint32(0x9E3779B9)
_PHILOX_W1 = np.uint32(0xBB67AE85)
_MASK32 = np.uint64(0xFFFFFFFF)

IH4_SCALE = 1.7320508075688772 / 4294967296.0   # sqrt(3) / 2^32, a double constant
IH4_CENTRE = (1 << 33) - 2                       # 4 * (2^32 - 1) / 2
OUTLIER_THRESHOLD = 4294967                      # u < this: ~0.1% of draws
OUTLIER_FACTOR = 100.0
MASTER_SIGMA = 0.02
WEIGHT_SIGMA = 0.02
GSCALE_LO, GSCALE_HI = np.float32(1e-5), np.float32(1e-2)
M_SPAN = np.float32(1e-3)   # |m| in [s_g * 1e-3, s_g]
V_SPAN = np.float32(0.1)    # v in [s_g^2 * 0.1, s_g^2]


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds on uint32 arrays (broadcasting)."""
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint32) for c in (c0, c1, c2, c3))
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    k0 = np.uint32(k0)
    k1 = np.uint32(k1)
    with np.errstate(over="ignore"):
        for _ in range(10):
            p0 = _PHILOX_M0 * c0.astype(np.uint64)
            p1 = _PHILOX_M1 * c2.astype(np.uint64)
            hi0 = (p0 >> np.uint64(32)).astype(np.uint32)
            lo0 = (p0 & _MASK32).astype(np.uint32)
            hi1 = (p1 >> np.uint64(32)).astype(np.uint32)
            lo1 = (p1 & _MASK32).astype(np.uint32)
            c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
            k0 = np.uint32(k0 + _PHILOX_W0)
            k1 = np.uint32(k1 + _PHILOX_W1)
    return c0, c1, c2, c3


def _draw(seed, stream, idx, tensor, step):
    idx = np.asarray(idx, dtype=np.int64)
    lo = (idx & 0xFFFFFFFF).astype(np.uint32)
    hi = (idx >> 32).astype(np.uint32)
    return philox4x32_10(lo, hi, np.uint32(tensor), np.uint32(step), np.uint32(seed), np.uint32(stream))


def _ih4(u0, u1, u2, u3):
    s = u0.astype(np.int64) + u1.astype(np.int64) + u2.astype(np.int64) + u3.astype(np.int64)
    return (s - IH4_CENTRE).astype(np.float64) * IH4_SCALE


def _bits(x):
    return np.asarray(x, dtype=np.float32).view(np.uint32)


def _loguniform(u, lo, hi):
    """Uniform over FP32 bit patterns in [bits(lo), bits(hi)); lo, hi > 0."""
    lb = _bits(lo).astype(np.uint64)
    hb = _bits(hi).astype(np.uint64)
    off = (u.astype(np.uint64) * (hb - lb)) >> np.uint64(32)
    return (lb + off).astype(np.uint32).view(np.float32)


def f32_to_bf16_bits(x):
    """Round-to-nearest-even FP32 -> bf16 bit patterns (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b):
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _idx(start, count):
    return np.arange(start, start + count, dtype=np.int64)


# ----------------------------------------------------------------------------
# Host generator
# ----------------------------------------------------------------------------

def master(seed, tensor, start, count):
    u = _draw(seed, MASTER, _idx(start, count), tensor, 0)
    return (MASTER_SIGMA * _ih4(*u)).astype(np.float32)


def group_scale(seed, tensor, gstart, gcount):
    u = _draw(seed, GSCALE, _idx(gstart, gcount), tensor, 0)
    return _loguniform(u[0], GSCALE_LO, GSCALE_HI)


def _scale_of(seed, tensor, start, count, group):
    g0 = start // group
    g1 = (start + count - 1) // group + 1 if count > 0 else g0
    sg = group_scale(seed, tensor, g0, g1 - g0)
    return sg[(_idx(start, count) // group) - g0]


def grad_bits(seed, tensor, step, start, count, group=128):
    u = _draw(seed, GRAD, _idx(start, count), tensor, step)
    sg = _scale_of(seed, tensor, start, count, group)
    return f32_to_bf16_bits((sg.astype(np.float64) * _ih4(*u)).astype(np.float32))


def m_warm(seed, tensor, start, count, group=128):
    u = _draw(seed, MSTATE, _idx(start, count), tensor, 0)
    sg = _scale_of(seed, tensor, start, count, group)
    mag = _loguniform(u[0], sg * M_SPAN, sg)
    return np.where((u[1] >> np.uint32(31)) != 0, -mag, mag).astype(np.float32)


def v_warm(seed, tensor, start, count, group=128):
    u = _draw(seed, VSTATE, _idx(start, count), tensor, 0)
    sg = _scale_of(seed, tensor, start, count, group)
    sg2 = (sg * sg).astype(np.float32)
    return _loguniform(u[0], sg2 * V_SPAN, sg2)


def activations_bits(seed, tensor, start, count):
    idx = _idx(start, count)
    u = _draw(seed, ACT, idx, tensor, 0)
    o = _draw(seed, ACT_OUTLIER, idx, tensor, 0)[0]
    z = _ih4(*u)
    z = np.where(o < np.uint32(OUTLIER_THRESHOLD), z * OUTLIER_FACTOR, z)
    return f32_to_bf16_bits(z.astype(np.float32))


def weight_bits(seed, tensor, start, count):
    u = _draw(seed, WEIGHT, _idx(start, count), tensor, 0)
    return f32_to_bf16_bits((WEIGHT_SIGMA * _ih4(*u)).astype(np.float32))


# ----------------------------------------------------------------------------
# Stored-state inputs: FP8 codes and per-group (k, scale) drawn directly, so
# that two implementations can start a step from bit-identical states.  Codes
# are uniform over the magnitudes an expanded group occupies (E4M3 0x01-0x7E,
# i.e. 2^-9..448; E5M2 0x34-0x7B, i.e. 0.25..57344), m with a random sign.
# k_m in [1.5, 2.2) (a group span of ~200..5000), root scale s_m = s_g *
# [0.02, 0.06) (largest |m| ~ s_g); k_v in [4, 8) (span ~5..22), s_v = s_g^2 *
# [0.1, 0.3).  `step` selects an independent draw per step.
# ----------------------------------------------------------------------------
CODE_RANGE = {0: (0x01, 0x7E), 1: (0x34, 0x7B), 2: (0x01, 0x7B)}   # E5M2 full span: 2^-16..57344


def _unit24(u):
    """[0, 1) FP32 from the top 24 bits (exact)."""
    return (u >> np.uint32(8)).astype(np.float32) * np.float32(2.0 ** -24)


def state_codes(seed, tensor, step, start, count, fmt, signed):
    lo, hi = CODE_RANGE[fmt]
    u = _draw(seed, MCODE if signed else VCODE, _idx(start, count), tensor, step)
    mag = (np.uint32(lo) + u[0] % np.uint32(hi - lo + 1)).astype(np.uint8)
    if signed:
        mag = mag | np.where((u[1] >> np.uint32(31)) != 0, 0x80, 0).astype(np.uint8)
    return mag


def state_groups(seed, tensor, step, gstart, gcount):
    """(k_m, s_m, k_v, s_v) float32 arrays for groups gstart.. of a tensor."""
    u = _draw(seed, GSTATE, _idx(gstart, gcount), tensor, step)
    sg = group_scale(seed, tensor, gstart, gcount)
    f = np.float32
    k_m = (f(0.7) * _unit24(u[0])).astype(np.float32) + f(1.5)
    s_m = sg * ((f(0.04) * _unit24(u[1])).astype(np.float32) + f(0.02))
    k_v = (f(4.0) * _unit24(u[2])).astype(np.float32) + f(4.0)
    sg2 = (sg * sg).astype(np.float32)
    s_v = sg2 * ((f(0.2) * _unit24(u[3])).astype(np.float32) + f(0.1))
    return (k_m.astype(np.float32), s_m.astype(np.float32), k_v.astype(np.float32),
            s_v.astype(np.float32))


# ----------------------------------------------------------------------------
# Device generator (CUDA, csrc/synth.cu) -- same numbers, written into
# caller-owned device buffers.
# ----------------------------------------------------------------------------

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcoat_synth.so")
_dlib = None


def device_lib():
    global _dlib
    if _dlib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("device input generator not built (%s); run __graft_entry__.build()" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32
        for name in ("synth_master", "synth_m_warm", "synth_v_warm", "synth_activations",
                     "synth_weight"):
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = [vp, i64, u32, u32, i64, vp]
        L.synth_grad.restype = ctypes.c_int
        L.synth_grad.argtypes = [vp, i64, u32, u32, u32, i64, vp]
        L.synth_state_codes.restype = ctypes.c_int
        L.synth_state_codes.argtypes = [vp, i64, u32, u32, u32, i64, ctypes.c_int, ctypes.c_int, vp]
        L.synth_state_groups.restype = ctypes.c_int
        L.synth_state_groups.argtypes = [vp, vp, vp, vp, i64, u32, u32, u32, i64, vp]
        _dlib = L
    return _dlib


def _stream_ptr(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(rc, what):
    if rc != 0:
        raise RuntimeError("%s failed (cuda error %d)" % (what, rc))


def device_master(out, seed, tensor, start=0, stream=None):
    """Fill a float32 CUDA tensor with master(seed, tensor, start, out.numel())."""
    _check(device_lib().synth_master(out.data_ptr(), out.numel(), seed, tensor, start,
                                     _stream_ptr(stream)), "synth_master")


def device_grad(out, seed, tensor, step, start=0, stream=None):
    """Fill a bf16/int16 CUDA tensor with grad_bits(...)."""
    _check(device_lib().synth_grad(out.data_ptr(), out.numel(), seed, tensor, step, start,
                                   _stream_ptr(stream)), "synth_grad")


def device_m_warm(out, seed, tensor, start=0, stream=None):
    _check(device_lib().synth_m_warm(out.data_ptr(), out.numel(), seed, tensor, start,
                                     _stream_ptr(stream)), "synth_m_warm")


def device_v_warm(out, seed, tensor, start=0, stream=None):
    _check(device_lib().synth_v_warm(out.data_ptr(), out.numel(), seed, tensor, start,
                                     _stream_ptr(stream)), "synth_v_warm")


def device_activations(out, seed, tensor, start=0, stream=None):
    _check(device_lib().synth_activations(out.data_ptr(), out.numel(), seed, tensor, start,
                                          _stream_ptr(stream)), "synth_activations")


def device_weight(out, seed, tensor, start=0, stream=None):
    _check(device_lib().synth_weight(out.data_ptr(), out.numel(), seed, tensor, start,
                                     _stream_ptr(stream)), "synth_weight")


def device_state_codes(out, seed, tensor, step, fmt, signed, start=0, stream=None):
    """Fill a uint8 CUDA tensor with state_codes(...)."""
    _check(device_lib().synth_state_codes(out.data_ptr(), out.numel(), seed, tensor, step, start,
                                          fmt, int(bool(signed)), _stream_ptr(stream)),
           "synth_state_codes")


def device_state_groups(k_m, s_m, k_v, s_v, seed, tensor, step, gstart=0, stream=None):
    """Fill four float32 CUDA tensors (one entry per group) with state_groups(...)."""
    _check(device_lib().synth_state_groups(k_m.data_ptr(), s_m.data_ptr(), k_v.data_ptr(),
                                           s_v.data_ptr(), k_m.numel(), seed, tensor, step, gstart,
                                           _stream_ptr(stream)), "synth_state_groups")
