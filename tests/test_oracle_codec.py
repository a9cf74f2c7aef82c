"""Pins for the oracle's per-group quantiser with dynamic range expansion.

The expansion formula (lost from the COAT pages' extracted text, page
"FP8训练新范式：减少40%显存占用，训练速度提高1.4倍", section
"解决方案：动态范围扩展") is fixed by the problem statement:
f(x) = sign(x)|x|^k, k = clamp(ln(448/2^-9) / ln(max/min_nonzero), 1, 16).
What pins the oracle's implementation of it, beyond itself:
  * the defining invariant: after expansion the group spans exactly 448/2^-9,
    its max lands on FMT_MAX and its min on FMT_MAX/R;
  * constructed groups whose expanded values are exact FP8 values must come
    back with exactly those codes and that k;
  * hand-derived 4-element examples (closed forms written out below);
  * the clamps and degenerate groups;
  * the page's error claims, by brute force on groups with its ratios.
"""
import math

import numpy as np
import pytest
import torch

E4M3, E5M2, E5M2_FULL = 0, 1, 2
R = 448.0 / 2.0 ** -9
R5 = 57344.0 / 2.0 ** -16   # E5M2's own span (the full-span reading)
FMAX = {E4M3: 448.0, E5M2: 57344.0, E5M2_FULL: 57344.0}
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def tdec(fmt, codes):
    """Decode through torch (independent of the oracle)."""
    c = torch.from_numpy(np.asarray(codes, dtype=np.uint8).copy())
    return c.view(TORCH_DT[fmt]).to(torch.float64).numpy()


def loguniform_group(rng, n, ratio, sign=True):
    mag = np.exp(rng.uniform(0.0, math.log(ratio), n))
    mag[0], mag[1] = 1.0, ratio  # pin the exact max/min ratio
    mag /= ratio
    if sign:
        mag *= rng.choice([-1.0, 1.0], n)
    return mag


# ---------------------------------------------------------------------------
# T3: the defining invariant of the expansion
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("fmt", [E4M3, E5M2, E5M2_FULL])
def test_expanded_span_equals_target(orc, fmt):
    rng = np.random.default_rng(10)
    Rf = R5 if fmt == E5M2_FULL else R
    for ratio in [Rf ** (1 / 16) * 1.01, 3.0, 10.0, 100.0, 1000.0, 1e4, R * 0.999]:
        if ratio < Rf ** (1 / 16):
            continue                      # k would clamp at 16 (checked separately)
        x = loguniform_group(rng, 128, ratio) * 3e-4
        M, k, s = orc.group_params(x, True, fmt)
        a = np.abs(x)
        mu = a[a > 0].min()
        assert M == a.max()
        expect_k = math.log(Rf) / math.log(M / mu)
        assert abs(k - expect_k) <= 1e-6 * expect_k
        # expanded max / expanded min == the target span (k rounded to FP32: ~1e-6 relative)
        assert abs((M / mu) ** k / Rf - 1) < 2e-6 * max(1.0, k / 8)
        codes, k2, s2 = orc.quantize_group(x, True, fmt)
        assert (k2, s2) == (k, s)
        i_max, i_min = int(np.argmax(a)), int(np.argmin(np.where(a > 0, a, np.inf)))
        assert codes[i_max] & 0x7F == (0x7E if fmt == E4M3 else 0x7B)
        # min maps to FMT_MAX/R: 2^-9 (E4M3 code 0x01), 0.25 (E5M2 code 0x34), or
        # E5M2's own smallest value 2^-16 (code 0x01) with the full-span target
        assert codes[i_min] & 0x7F == {E4M3: 0x01, E5M2: 0x34, E5M2_FULL: 0x01}[fmt]
        # the root scale brings the max code back to M
        assert abs(s * FMAX[fmt] ** (1 / k) / M - 1) < 2e-7


def test_k_clamps(orc):
    x = np.array([1.0, 0.5, 0.9, -0.7])            # ratio 2 < R^(1/16) = 2.163 -> k = 16
    assert orc.group_params(x, True, E4M3)[1] == 16.0
    x = np.array([1.0, 1e-7, 0.3])                 # ratio 1e7 > R -> k = 1
    assert orc.group_params(x, True, E4M3)[1] == 1.0
    x = np.array([2.0, -2.0, 0.0, 2.0])            # one magnitude -> k = 16
    assert orc.group_params(x, True, E4M3)[1] == 16.0
    x = np.array([1.0, 1e-3])                      # expansion off -> k = 1
    M, k, s = orc.group_params(x, False, E4M3)
    assert (k, s) == (1.0, np.float32(1.0 / 448.0))


# ---------------------------------------------------------------------------
# T4: constructed groups that sit exactly on FP8 values round-trip exactly
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_constructed_group_recovers_codes(orc, fmt):
    rng = np.random.default_rng(11)
    top = 0x7E if fmt == E4M3 else 0x7B
    lo_code = 0x01 if fmt == E4M3 else 0x34   # the code of FMT_MAX / R
    for k0 in [1.0, 1.5, 2.680274, 5.4, 9.0, 15.5]:
        codes = rng.integers(lo_code, top + 1, 128).astype(np.uint8)
        codes[0], codes[1] = top, lo_code
        codes |= rng.choice([0, 0x80], 128).astype(np.uint8)
        M = 7.5e-3
        y = np.abs(tdec(fmt, codes))
        x = M * (y / FMAX[fmt]) ** (1.0 / k0) * np.where(codes & 0x80, -1.0, 1.0)
        q, k, s = orc.quantize_group(x, True, fmt)
        assert abs(k - k0) <= 1e-6 * k0
        assert np.array_equal(q, codes)
        xr = np.array([orc.dequant_value(fmt, c, s, k) for c in q])
        assert np.allclose(xr, x, rtol=2e-6, atol=0)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_roundtrip_error_bound(orc, fmt):
    """|dequant(quant(x)) - x| is bounded by half an FP8 step, mapped back through
    the 1/k power, for every element the expansion puts in the normal range."""
    rng = np.random.default_rng(12)
    half_ulp_rel = 2.0 ** -4 if fmt == E4M3 else 2.0 ** -3
    min_normal = 2.0 ** -6 if fmt == E4M3 else 2.0 ** -14
    for ratio in (10.0, 1000.0):
        for _ in range(20):
            x = loguniform_group(rng, 128, ratio) * 1e-3
            q, k, s = orc.quantize_group(x, True, fmt)
            xr = np.array([orc.dequant_value(fmt, c, s, k) for c in q])
            y = FMAX[fmt] * (np.abs(x) / np.abs(x).max()) ** k
            normal = y >= min_normal
            bound = ((1 + half_ulp_rel) ** (1 / k) - 1) * np.abs(x) * (1 + 1e-6)
            assert np.all(np.abs(xr - x)[normal] <= bound[normal])
            assert np.all(np.sign(xr[xr != 0]) == np.sign(x[xr != 0]))


# ---------------------------------------------------------------------------
# T5: hand-derived worked examples (group of 4; closed forms in comments)
# ---------------------------------------------------------------------------
def test_worked_example_e4m3(orc):
    # x = [1, -0.1, 0.01, 0]: M = 1, mu = 0.01, so k = ln R / ln 100.
    # y(1) = 448 -> 0x7E.  y(0.1) = 448 * 0.1^k = 448 / sqrt(R) = 0.93541, between
    # 0.875 (0x36) and 0.9375 (0x37), midpoint 0.90625 -> 0x37, negative -> 0xB7.
    # y(0.01) = 448 / R = 2^-9 -> 0x01.
    x = [1.0, -0.1, 0.01, 0.0]
    q, k, s = orc.quantize_group(x, True, E4M3)
    k_exact = math.log(R) / math.log(100.0)
    assert abs(k - k_exact) < 1e-6 * k_exact
    assert list(q) == [0x7E, 0xB7, 0x01, 0x00]
    # s_r = 448^(-1/k): dequant of 0x7E is 1, of 0x01 is R^(-1/k) = 0.01
    assert abs(s - 448.0 ** (-1 / k_exact)) < 1e-7
    xr = [orc.dequant_value(E4M3, c, s, k) for c in q]
    assert abs(xr[0] - 1.0) < 1e-7
    assert abs(xr[1] + (0.9375 / 448.0) ** (1 / k_exact)) < 1e-7   # = -0.1000831...
    assert abs(xr[1] + 0.10008313) < 1e-7
    assert abs(xr[2] - 0.01) < 1e-8
    assert xr[3] == 0.0


def test_worked_example_e5m2_and_small_ratio(orc):
    # Same x in E5M2 (target range still R): y = 57344 (0x7B), 57344/sqrt(R) =
    # 119.73 between 112 (0x57) and 128 (0x58), midpoint 120 -> 0x57 -> 0xD7;
    # 57344 / R = 0.25 -> 0x34.
    q, k, s = orc.quantize_group([1.0, -0.1, 0.01, 0.0], True, E5M2)
    assert list(q) == [0x7B, 0xD7, 0x34, 0x00]
    # x = [4e-6, 1e-6, -0, 2e-6]: ratio 4, k = ln R / ln 4 = 8.9037.
    # y(1e-6) = 448 / R = 2^-9 -> 0x01; y(2e-6) = 448 * 2^-k = 448/sqrt(R) -> 0x37.
    q, k, s = orc.quantize_group([4e-6, 1e-6, -0.0, 2e-6], True, E4M3)
    assert abs(k - math.log(R) / math.log(4.0)) < 1e-5
    assert list(q) == [0x7E, 0x01, 0x00, 0x37]


def test_worked_example_no_expansion(orc):
    # k = 1, s_r = 1/448: y = 448|x| -> 448 (0x7E); 44.8 between 44 (0 1100 011 = 0x63)
    # and 48 (0x64) -> 0x63, negative 0xE3; 4.48 between 4.0 (0x48) and 4.5 (0x49) -> 0x49.
    q, k, s = orc.quantize_group([1.0, -0.1, 0.01, 0.0], False, E4M3)
    assert (k, s) == (1.0, np.float32(1 / 448))
    assert list(q) == [0x7E, 0xE3, 0x49, 0x00]
    assert list(tdec(E4M3, q)) == [448.0, -44.0, 4.5, 0.0]


# ---------------------------------------------------------------------------
# T6: degenerate groups
# ---------------------------------------------------------------------------
def test_degenerate_groups(orc):
    q, k, s = orc.quantize_group(np.zeros(128), True, E4M3)
    assert (k, s) == (1.0, 1.0) and not q.any()
    x = np.zeros(128)
    x[17] = -3.5
    q, k, s = orc.quantize_group(x, True, E4M3)
    assert k == 16.0 and q[17] == 0xFE and np.count_nonzero(q) == 1
    assert abs(orc.dequant_value(E4M3, q[17], s, k) + 3.5) < 3.5e-7
    x = np.full(128, 0.25)
    x[::3] *= -1
    q, k, s = orc.quantize_group(x, True, E5M2)
    assert k == 16.0 and set(q) == {0x7B, 0xFB}


def test_2d_blocks_and_ragged_edges(orc):
    rng = np.random.default_rng(13)
    x = rng.standard_normal((300, 200)) * np.exp(rng.uniform(-3, 3, (300, 200)))
    for gr, gc in ((1, 128), (128, 128)):
        q, s, k = orc.group_quantize(x, gr, gc, True, E4M3)
        assert s.shape == (-(-300 // gr), -(-200 // gc))
        for bi in range(s.shape[0]):
            for bj in range(s.shape[1]):
                blk = x[bi * gr:(bi + 1) * gr, bj * gc:(bj + 1) * gc]
                qq, kk, ss = orc.quantize_group(blk.ravel(), True, E4M3)
                assert np.array_equal(q[bi * gr:(bi + 1) * gr, bj * gc:(bj + 1) * gc].ravel(), qq)
                assert (k[bi, bj], s[bi, bj]) == (np.float32(kk), np.float32(ss))
        xr = orc.group_dequantize(q, s, k, gr, gc, E4M3)
        assert xr.shape == x.shape
        assert np.all(np.sign(xr[xr != 0]) == np.sign(x[xr != 0]))


# ---------------------------------------------------------------------------
# T7: the page's error claims, by brute force
# ---------------------------------------------------------------------------
def _mse(orc, groups, fmt, expand):
    err = 0.0
    for x in groups:
        q, k, s = orc.quantize_group(x, expand, fmt)
        xr = np.array([orc.dequant_value(fmt, c, s, k) for c in q])
        err += float(np.mean((xr - x) ** 2))
    return err / len(groups)


def test_e5m2_matches_e4m3_for_v_only_with_its_own_span(orc):
    """Same section: after expansion E4M3 and E5M2 are almost the same for the
    second moment.  With the literal target 448 / 2^-9 E5M2's error stays
    several times E4M3's; expanding to E5M2's own span 57344 / 2^-16 brings it
    to within a few percent of E4M3's."""
    rng = np.random.default_rng(15)
    v_groups = [loguniform_group(rng, 128, 10.0, sign=False) * 1e-6 for _ in range(60)]
    e4 = _mse(orc, v_groups, E4M3, True)
    e5 = _mse(orc, v_groups, E5M2, True)
    e5f = _mse(orc, v_groups, E5M2_FULL, True)
    assert e5 > 2.0 * e4
    assert abs(e5f / e4 - 1.0) < 0.25
    # and the full-span k is larger: the group is stretched over more binades
    k4 = orc.group_params(v_groups[0], True, E4M3)[1]
    k5f = orc.group_params(v_groups[0], True, E5M2_FULL)[1]
    assert abs(k5f / k4 - math.log(R5) / math.log(R)) < 1e-6


def test_expansion_reduces_error_on_pages_ratios(orc):
    """Page "FP8训练新范式", section "解决方案：动态范围扩展": expansion greatly
    reduces quantisation error; E4M3 suits the first moment better than E5M2;
    without expansion E4M3 beats E5M2 for the second moment."""
    rng = np.random.default_rng(14)
    m_groups = [loguniform_group(rng, 128, 1000.0) * 1e-3 for _ in range(60)]
    v_groups = [loguniform_group(rng, 128, 10.0, sign=False) * 1e-6 for _ in range(60)]
    mse = {}
    for name, groups in (("m", m_groups), ("v", v_groups)):
        for fmt in (E4M3, E5M2):
            for expand in (False, True):
                mse[name, fmt, expand] = _mse(orc, groups, fmt, expand)
    for name in ("m", "v"):
        for fmt in (E4M3, E5M2):
            assert mse[name, fmt, True] < 0.5 * mse[name, fmt, False], (name, fmt)
    assert mse["m", E4M3, True] < mse["m", E5M2, True]
    assert mse["m", E4M3, False] < mse["m", E5M2, False]
    assert mse["v", E4M3, False] < mse["v", E5M2, False]
