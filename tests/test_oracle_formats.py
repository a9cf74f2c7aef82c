"""Pins for the oracle's FP8 formats and encoder.

Decode: checked against the values the COAT pages print (E4M3 spans 0.00195 to
448, a dynamic range of about 200000 -- page "FP8训练新范式：减少40%显存占用，
训练速度提高1.4倍", section "FP8优化器状态"), against the 1+4+3 / 1+5+2 bit
layouts (page "FP8量化训练实战指南", section "格式选择：E4M3与E5M2的智能搭配"),
and against torch's own float8_e4m3fn / float8_e5m2 decoding, a library routine
independent of the oracle.

Encode: checked against brute-force nearest search done here with numpy over
torch's decode table, against torch's float8 casts on in-range values, and at
every rounding midpoint.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_constants.json")
E4M3, E5M2 = 0, 1
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def torch_decode_table(fmt):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(TORCH_DT[fmt]).to(torch.float64).numpy()


def same_or_both_nan(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return bool(np.all((a == b) | (np.isnan(a) & np.isnan(b))))


@pytest.fixture(scope="module")
def pages():
    with open(GOLDEN) as f:
        return json.load(f)


def test_decode_matches_torch_all_codes(orc):
    for fmt in (E4M3, E5M2):
        mine = orc.fp8_decode_table(fmt)
        ref = torch_decode_table(fmt)
        assert same_or_both_nan(mine, ref), fmt


def test_e4m3_printed_constants(orc, pages):
    t = orc.fp8_decode_table(E4M3)
    pos = t[1:128][np.isfinite(t[1:128])]
    lo, hi = pos.min(), pos.max()
    assert hi == pages["e4m3_max_representable"]
    # the page prints 0.00195 (3 significant digits)
    assert round(lo, 5) == pages["e4m3_min_representable"]
    assert lo == 2.0 ** -9
    rng = hi / lo
    assert rng == 229376.0
    # "about 200000": within the page's one-significant-digit precision
    assert abs(rng - pages["e4m3_dynamic_range_approx"]) / pages["e4m3_dynamic_range_approx"] < 0.2
    assert orc.target_range() == rng
    assert orc.target_range(1) == rng                       # E5M2: the same literal span
    assert orc.target_range(2) == 57344.0 * 2.0 ** 16          # E5M2's own span
    # the group ratios the page reports are far below that range
    assert pages["first_moment_group_max_min_ratio_typical"] < rng
    assert pages["second_moment_group_max_min_ratio_typical"] < rng


def test_bit_layouts(orc, pages):
    # E4M3: 1 sign + 4 exponent + 3 mantissa, bias 7; 1.0 = 0 0111 000
    assert pages["e4m3_bits"] == {"sign": 1, "exponent": 4, "mantissa": 3}
    assert orc.fp8_decode(E4M3, 0b0_0111_000) == 1.0
    assert orc.fp8_decode(E4M3, 0b0_0111_001) == 1.125
    assert orc.fp8_decode(E4M3, 0b1_1000_100) == -3.0
    assert orc.fp8_decode(E4M3, 0b0_0001_000) == 2.0 ** -6     # smallest normal
    assert orc.fp8_decode(E4M3, 0b0_0000_111) == 7 * 2.0 ** -9  # largest subnormal
    assert math.isnan(orc.fp8_decode(E4M3, 0x7F)) and math.isnan(orc.fp8_decode(E4M3, 0xFF))
    assert all(np.isfinite(orc.fp8_decode_table(E4M3)[[c for c in range(256) if c & 0x7F != 0x7F]]))
    # E5M2: 1 + 5 + 2, bias 15; 1.0 = 0 01111 00
    assert pages["e5m2_bits"] == {"sign": 1, "exponent": 5, "mantissa": 2}
    assert orc.fp8_decode(E5M2, 0b0_01111_00) == 1.0
    assert orc.fp8_decode(E5M2, 0b0_01111_01) == 1.25
    assert orc.fp8_decode(E5M2, 0x7B) == 57344.0
    assert orc.fp8_decode(E5M2, 0x01) == 2.0 ** -16
    assert orc.fp8_decode(E5M2, 0x7C) == math.inf and orc.fp8_decode(E5M2, 0xFC) == -math.inf
    for c in (0x7D, 0x7E, 0x7F):
        assert math.isnan(orc.fp8_decode(E5M2, c))


def test_positive_codes_increase(orc):
    for fmt, top in ((E4M3, 0x7E), (E5M2, 0x7B)):
        t = orc.fp8_decode_table(fmt)[: top + 1]
        assert np.all(np.diff(t) > 0)
        neg = orc.fp8_decode_table(fmt)[128: 128 + top + 1]
        assert np.array_equal(neg[1:], -t[1:])


def brute_nearest(fmt, y):
    """Nearest finite code to each FP32 value, ties to the even code, saturating --
    written here directly from the definition over torch's decode table."""
    table = torch_decode_table(fmt)
    top = 0x7E if fmt == E4M3 else 0x7B
    mags = table[: top + 1]
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(y), mags[-1])
    d = np.abs(mags[None, :] - a[:, None])
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    even = cand & (np.arange(top + 1)[None, :] % 2 == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    sign = np.where(np.signbit(y) & (pick != 0), 0x80, 0)
    return (pick | sign).astype(np.uint8)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encode_matches_brute_force(orc, fmt):
    rng = np.random.default_rng(1)
    top = 448.0 if fmt == E4M3 else 57344.0
    lo = 2.0 ** -12 if fmt == E4M3 else 2.0 ** -19
    mag = np.exp(rng.uniform(np.log(lo), np.log(top * 1.2), 20000))
    y = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32)
    y = np.concatenate([y, np.float32([0.0, -0.0, top, -top, top * 2, 1e30, -1e30])])
    got = orc.fp8_encode_array(fmt, y)
    assert np.array_equal(got, brute_nearest(fmt, y))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encode_matches_torch_cast_in_range(orc, fmt):
    rng = np.random.default_rng(2)
    top = 448.0 if fmt == E4M3 else 57344.0
    y = rng.uniform(-top, top, 50000).astype(np.float32)
    y[:5000] *= 1e-3
    y[5000:10000] *= 1e-5
    got = orc.fp8_encode_array(fmt, y)
    ref = torch.from_numpy(y).to(TORCH_DT[fmt]).view(torch.uint8).numpy().copy()
    ref[ref == 0x80] = 0  # this library writes every zero magnitude as code 0x00
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encode_midpoints_round_to_even(orc, fmt):
    top = 0x7E if fmt == E4M3 else 0x7B
    t = torch_decode_table(fmt)[: top + 1]
    for c in range(top):
        mid = np.float32((t[c] + t[c + 1]) / 2)   # exact in FP32
        assert float(mid) == (t[c] + t[c + 1]) / 2
        even = c if c % 2 == 0 else c + 1
        assert orc.fp8_encode(fmt, float(mid)) == even
        up = np.nextafter(mid, np.float32(np.inf))
        dn = np.nextafter(mid, np.float32(-np.inf))
        assert orc.fp8_encode(fmt, float(up)) == c + 1
        assert orc.fp8_encode(fmt, float(dn)) == c
        if c + 1 <= top:
            assert orc.fp8_encode(fmt, float(-up)) == 0x80 | (c + 1)


def test_encode_special_values(orc):
    assert orc.fp8_encode(E4M3, 2.0 ** -10) == 0          # tie between 0 and 2^-9 -> even code 0
    assert orc.fp8_encode(E4M3, float(np.nextafter(np.float32(2 ** -10), np.float32(1)))) == 1
    assert orc.fp8_encode(E4M3, -1e-6) == 0               # negative magnitude zero -> 0x00
    assert orc.fp8_encode(E4M3, -0.0) == 0
    for y in (449.0, 464.0, 465.0, 479.0, 480.0, 1e38, math.inf):
        assert orc.fp8_encode(E4M3, y) == 0x7E
        assert orc.fp8_encode(E4M3, -y) == 0xFE
    for y in (57345.0, 61440.0, 61441.0, 1e38, math.inf):
        assert orc.fp8_encode(E5M2, y) == 0x7B
    assert orc.fp8_encode(E4M3, math.nan) & 0x7F == 0x7F
    assert orc.fp8_encode(E5M2, math.nan) & 0x7F == 0x7F
    assert orc.fp8_encode(E5M2, 2.0 ** -17) == 0          # tie between 0 and 2^-16
    assert orc.fp8_encode(E5M2, 0.25) == 0x34


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    mine = orc.float_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)
