"""Exact checks of two small arithmetic steps the codec kernels rely on,
restated in rational arithmetic on the CPU (no GPU, no library code).

* The bf16 quantiser paths take RN(1/b) for a group maximum b (a bf16 value,
  possibly scaled by 2^64) as one Newton step y1 = RN(y0 + y0 RN(1 - b y0))
  from the hardware's approximate reciprocal y0, which is within one ulp of
  1/b.  The step must give RN(1/b) for every such seed: checked for all 128
  bf16 significands and both neighbours of 1/b.  The RMSNorm forward does the
  same for products of an FP8 value and a bf16 value: all 2048 significands
  of at most 12 bits.
* The root scale M / FMT_MAX is taken as q1 = RN(q0 + r y) with y = RN(1/FMT_MAX),
  q0 = RN(M y), r = RN(M - q0 FMT_MAX) (the division's correction step).  It
  must equal RN(M / FMT_MAX): checked for every bf16 significand and, for
  FP32 inputs, on 20,000 seeded significands per format.
"""
import math
import random
from fractions import Fraction as Fr

import pytest


def _binade(x):
    e = math.floor(math.log2(x))
    while Fr(2) ** e > x:
        e -= 1
    while Fr(2) ** (e + 1) <= x:
        e += 1
    return e


def rn32(x):
    """x rounded to FP32 (normal range), ties to even."""
    if x == 0:
        return Fr(0)
    if x < 0:
        return -rn32(-x)
    q = Fr(2) ** (_binade(x) - 23)
    n = x / q
    f = math.floor(n)
    r = n - f
    if r > Fr(1, 2) or (r == Fr(1, 2) and f % 2 == 1):
        f += 1
    return f * q


def ulp32(x):
    return Fr(2) ** (_binade(abs(x)) - 23)


def fma(a, b, c):
    return rn32(a * b + c)


def seeds_within_ulp(b):
    """The FP32 values less than one ulp from 1/b (the reciprocal
    approximation's documented bound)."""
    want = rn32(1 / b)
    cands = (want - ulp32(want), want, want + ulp32(want))
    return [y for y in cands if abs(y - 1 / b) < ulp32(1 / b)]


@pytest.mark.parametrize("scale_exp", [0, 64 - 130, 100])
def test_newton_reciprocal_is_correctly_rounded_for_bf16_significands(scale_exp):
    bad = []
    for m in range(128):
        b = (1 + Fr(m, 128)) * Fr(2) ** scale_exp
        want = rn32(1 / b)
        for seed in seeds_within_ulp(b):
            got = fma(fma(-b, seed, Fr(1)), seed, seed)
            if got != want:
                bad.append((m, seed))
    assert not bad


def test_newton_reciprocal_is_correctly_rounded_for_12_bit_significands():
    # the RMSNorm forward's group maximum max|f w| is a product of an FP8 value
    # (at most 4 significant bits) and a bf16 weight (8 bits): at most 12 bits,
    # every one of which is covered here
    bad = []
    for m in range(2048):
        b = 1 + Fr(m, 2048)
        want = rn32(1 / b)
        for seed in seeds_within_ulp(b):
            if fma(fma(-b, seed, Fr(1)), seed, seed) != want:
                bad.append((m, seed))
    assert not bad


def test_newton_reciprocal_is_not_exact_in_general():
    # with 24-bit significands one step can miss RN(1/b): the all-ones
    # significand 2 - 2^-23 is a case, so the bf16 test above states a
    # property of short significands, not of the step in general
    b = 2 - Fr(1, 1 << 23)
    want = rn32(1 / b)
    assert any(fma(fma(-b, seed, Fr(1)), seed, seed) != want for seed in seeds_within_ulp(b))


@pytest.mark.parametrize("fmax", [448, 57344])
def test_root_scale_correction_step(fmax):
    fmax = Fr(fmax)
    y = rn32(1 / fmax)
    rng = random.Random(11)
    sigs = [1 + Fr(m, 128) for m in range(128)]
    sigs += [1 + Fr(rng.randrange(1 << 23), 1 << 23) for _ in range(20000)]
    bad = 0
    for s in sigs:
        for e in (-90, -3, 0, 7, 100):
            M = s * Fr(2) ** e
            q0 = rn32(M * y)
            r = fma(-q0, fmax, M)
            assert r == M - q0 * fmax          # the remainder is exact
            if fma(r, y, q0) != rn32(M / fmax):
                bad += 1
    assert bad == 0
