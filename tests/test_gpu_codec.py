"""GPU parity of the FP8 element codec and the per-group quantiser (1x128 and
128x128, expansion on/off) against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import fp8_optimizer_state_b200 as coat
import synth
from tests.parity import compare_codes, rel_err, scale_rtol, K_RTOL, FLIP_FRACTION

pytestmark = pytest.mark.gpu
E4M3, E5M2, E5M2_FULL = 0, 1, 2
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def encoder_probe_values():
    """Every FP32 exponent; for each, all 2^12 combinations of the top 12 mantissa
    bits with the low 11 bits at 0, 1 and all-ones -- which covers, for both
    formats, every rounding midpoint and its two FP32 neighbours -- both signs,
    plus NaN and infinities."""
    e = np.arange(256, dtype=np.uint32)[:, None, None]
    top = np.arange(4096, dtype=np.uint32)[None, :, None]
    low = np.array([0, 1, 0x7FF], dtype=np.uint32)[None, None, :]
    bits = ((e << np.uint32(23)) | (top << np.uint32(11)) | low).ravel()
    bits = np.concatenate([bits, bits | np.uint32(0x80000000)])
    return bits.view(np.float32)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encoder_bit_identical_to_oracle(orc, fmt):
    y = encoder_probe_values()
    q = torch.empty(y.size, dtype=torch.uint8, device="cuda")
    coat.coat_fp8_encode(torch.from_numpy(y).cuda(), fmt, q)
    got = q.cpu().numpy()
    ref = orc.fp8_encode_array(fmt, y)
    nan = np.isnan(y)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.all(got[nan] & 0x7F == 0x7F)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encoder_matches_hardware_cast_in_range(fmt):
    top = 448.0 if fmt == E4M3 else 57344.0
    g = torch.Generator(device="cuda").manual_seed(5)
    y = (torch.rand(1 << 22, device="cuda", generator=g) * 2 - 1) * top
    y[: 1 << 20] *= 1e-3
    q = torch.empty(y.numel(), dtype=torch.uint8, device="cuda")
    coat.coat_fp8_encode(y, fmt, q)
    ref = y.to(TORCH_DT[fmt]).view(torch.uint8).clone()
    ref[ref == 0x80] = 0
    assert torch.equal(q, ref)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encoder_exhaustive_up_to_format_max(fmt):
    """Every non-negative FP32 value up to FMT_MAX (1 + 2^-16) -- the range the
    step's expanded values take -- encodes as the hardware's round-to-nearest-
    even conversion does (about 1.1e9 values per format, in chunks)."""
    top = 448.0 if fmt == E4M3 else 57344.0
    last = int(np.float32(top * (1 + 2.0 ** -16)).view(np.uint32))
    chunk = 1 << 27
    q = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    for a in range(0, last + 1, chunk):
        n = min(chunk, last + 1 - a)
        y = torch.arange(a, a + n, dtype=torch.int64, device="cuda").to(torch.int32).view(torch.float32)
        coat.coat_fp8_encode(y, fmt, q[:n])
        ref = y.to(TORCH_DT[fmt]).view(torch.uint8)
        bad = (q[:n] != ref).nonzero()
        assert bad.numel() == 0, "y bits %#x: got %#x, want %#x" % (
            a + int(bad[0]), int(q[int(bad[0])]), int(ref[int(bad[0])]))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_decoder_all_codes(orc, fmt):
    q = torch.arange(256, dtype=torch.int32).to(torch.uint8).cuda()
    out = torch.empty(256, dtype=torch.float32, device="cuda")
    coat.coat_fp8_decode(q, fmt, out)
    got = out.cpu().numpy().astype(np.float64)
    ref = orc.fp8_decode_table(fmt)
    assert np.all((got == ref) | (np.isnan(got) & np.isnan(ref)))


def _check_quant(gq, gs, gk, oq, os_, ok_, fmt):
    assert rel_err(gk, ok_).max() <= K_RTOL
    assert np.all(rel_err(gs, os_) <= scale_rtol(ok_, fmt))
    diff, maxd = compare_codes(gq, oq)
    assert maxd <= 1
    assert diff.sum() <= max(1, FLIP_FRACTION * diff.size), int(diff.sum())


CASES = [(1, 128, 200, 1000), (1, 128, 64, 4096), (128, 128, 300, 260), (128, 128, 256, 384)]


@pytest.mark.parametrize("gr,gc,rows,cols", CASES)
@pytest.mark.parametrize("fmt", [E4M3, E5M2, E5M2_FULL])
@pytest.mark.parametrize("expand", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_group_quantize_vs_oracle(orc, gr, gc, rows, cols, fmt, expand, dtype):
    n = rows * cols
    ldx = -(-cols // 8) * 8          # rows padded to 16 bytes (the ABI's stride rule)
    if dtype == "bf16":
        bits = synth.activations_bits(0, rows + cols, 0, n).reshape(rows, cols)
        xh = synth.bf16_bits_to_f32(bits)
        xd = torch.zeros((rows, ldx), dtype=torch.int16, device="cuda")
        xd[:, :cols] = torch.from_numpy(bits.view(np.int16)).cuda()
    else:
        xh = (synth.master(0, rows + cols, 0, n) * np.float32(50.0)).reshape(rows, cols)
        xd = torch.zeros((rows, ldx), dtype=torch.float32, device="cuda")
        xd[:, :cols] = torch.from_numpy(xh).cuda()
    xd = xd[:, :cols]
    nbr, nbc = -(-rows // gr), -(-cols // gc)
    ldq = -(-cols // 16) * 16
    q = torch.zeros((rows, ldq), dtype=torch.uint8, device="cuda")
    s = torch.zeros((nbr, nbc), dtype=torch.float32, device="cuda")
    k = torch.zeros((nbr, nbc), dtype=torch.float32, device="cuda")
    coat.coat_group_quantize(xd, gr, gc, expand, fmt, q, s, k)
    oq, os_, ok_ = orc.group_quantize(xh.astype(np.float64), gr, gc, expand, fmt)
    torch.cuda.synchronize()
    _check_quant(q.cpu().numpy()[:, :cols], s.cpu().numpy(), k.cpu().numpy(), oq, os_, ok_, fmt)
    assert not q.cpu().numpy()[:, cols:].any()     # nothing written past cols
    if not expand:
        # k = 1: the root scale is M / FMT_MAX correctly rounded on both sides
        # (the oracle's double product rounds to the same FP32 value except in
        # double-rounding cases, about one in 2^29)
        assert np.array_equal(s.cpu().numpy(), os_)


@pytest.mark.parametrize("gr", [1, 128])
@pytest.mark.parametrize("fmt", [E4M3, E5M2, E5M2_FULL])
@pytest.mark.parametrize("expand", [False, True])
def test_group_quantize_special_values(orc, gr, fmt, expand):
    """Groups holding NaN or +-Inf follow the oracle: the maximum ignores NaN, a
    NaN element encodes as a NaN code, an Inf maximum gives k = 1 and an
    infinite scale with every finite element at code 0, and a group whose only
    values are NaN is all zeros with k = 1, scale 1.  Ordinary groups beside
    them are unaffected."""
    rows, cols = (4, 512) if gr == 1 else (256, 256)
    bits = synth.activations_bits(3, 7, 0, rows * cols).reshape(rows, cols)
    x = synth.bf16_bits_to_f32(bits).copy()
    nan, inf = np.float32(np.nan), np.float32(np.inf)
    if gr == 1:
        x[0, 5] = nan                  # group (0, 0): one NaN
        x[1, 130] = inf                # group (1, 1): +Inf
        x[2, 260], x[2, 300] = -inf, nan   # group (2, 2): -Inf and NaN
        x[3, 384:512] = nan            # group (3, 3): all NaN
    else:
        x[3, 5] = nan                  # block (0, 0)
        x[130, 7] = inf                # block (1, 0)
        x[20, 200], x[90, 129] = -inf, nan   # block (0, 1)
        x[128:, 128:] = nan            # block (1, 1): all NaN
    xb = torch.from_numpy(x).to(torch.bfloat16).cuda()
    nbr, nbc = -(-rows // gr), cols // 128
    q = torch.zeros((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.zeros((nbr, nbc), dtype=torch.float32, device="cuda")
    k = torch.zeros((nbr, nbc), dtype=torch.float32, device="cuda")
    coat.coat_group_quantize(xb, gr, 128, expand, fmt, q, s, k)
    oq, os_, ok_ = orc.group_quantize(xb.float().cpu().numpy().astype(np.float64), gr, 128,
                                      expand, fmt)
    gq, gs, gk = q.cpu().numpy(), s.cpu().numpy(), k.cpu().numpy()
    # exact groups: an Inf maximum, or NaN only (k = 1 and a scale of Inf or 1)
    exact = np.zeros((nbr, nbc), dtype=bool)
    xs = xb.float().cpu().numpy()
    for bi in range(nbr):
        for bj in range(nbc):
            blk = xs[bi * gr:(bi + 1) * gr, bj * 128:(bj + 1) * 128]
            exact[bi, bj] = np.isinf(blk).any() or np.isnan(blk).all()
    assert exact.sum() == 3
    assert np.array_equal(gk[exact], ok_[exact]) and np.array_equal(gs[exact], os_[exact])
    assert np.all(rel_err(gk[~exact], ok_[~exact]) <= K_RTOL)
    assert np.all(rel_err(gs[~exact], os_[~exact]) <= scale_rtol(ok_[~exact], fmt))
    el_exact = np.repeat(np.repeat(exact, gr, axis=0), 128, axis=1)[:rows]
    nan_code = (oq & 0x7F) == 0x7F
    assert nan_code.sum() >= 3
    assert np.all((gq[nan_code] & 0x7F) == 0x7F)              # NaN codes (sign may differ)
    same = el_exact & ~nan_code
    assert np.array_equal(gq[same], oq[same])
    rest = ~el_exact & ~nan_code
    diff, maxd = compare_codes(gq[rest], oq[rest])
    assert maxd <= 1 and diff.sum() <= max(1, FLIP_FRACTION * diff.size)


# Exponents of the power of two each row (1x128) or each 128-row block
# (128x128) is multiplied by: group maxima from 2^127.3 down to FP32
# subnormals, across the points where FMT_MAX |x| overflows (2^112-2^119), the
# approximate reciprocal flushes (2^126, 2^-126) and the 2^+-100 bounds of the
# range the kernels scale groups into.
EXTREME_EXPONENTS = [119, 116, 112, 105, 101, 100, 99, 0, -99, -100, -101, -110, -120, -126,
                     -130, -135]


@pytest.mark.parametrize("gr", [1, 128])
@pytest.mark.parametrize("fmt", [E4M3, E5M2, E5M2_FULL])
@pytest.mark.parametrize("expand", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_group_quantize_extreme_magnitudes(orc, gr, fmt, expand, dtype):
    """Groups of every magnitude FP32 holds follow the oracle (which divides in
    double and never overflows): k, the root scale (within its tolerance or one
    subnormal step, whichever is larger; bit-exact without expansion) and the
    codes."""
    ne = len(EXTREME_EXPONENTS)
    cols = 512
    rows = ne * gr
    bits = synth.activations_bits(4, rows + cols, 0, rows * cols).reshape(rows, cols)
    xv = synth.bf16_bits_to_f32(bits).astype(np.float64)
    xv *= np.repeat(2.0 ** np.array(EXTREME_EXPONENTS, dtype=np.float64), gr)[:, None]
    if dtype == "bf16":
        xd = torch.from_numpy(xv.astype(np.float32)).to(torch.bfloat16).cuda()
        xh = xd.float().cpu().numpy()
    else:
        xh = xv.astype(np.float32)
        xd = torch.from_numpy(xh).cuda()
    assert np.isfinite(xh).all()
    nbr, nbc = rows // gr, cols // 128
    q = torch.zeros((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.zeros((nbr, nbc), dtype=torch.float32, device="cuda")
    k = torch.zeros((nbr, nbc), dtype=torch.float32, device="cuda")
    coat.coat_group_quantize(xd, gr, 128, expand, fmt, q, s, k)
    oq, os_, ok_ = orc.group_quantize(xh.astype(np.float64), gr, 128, expand, fmt)
    gq, gs, gk = q.cpu().numpy(), s.cpu().numpy(), k.cpu().numpy()
    assert rel_err(gk, ok_).max() <= K_RTOL
    # the scale tolerance, but never below one subnormal step (2^-149): a
    # subnormal root scale keeps only the bits above it, on both sides
    tol = np.maximum(scale_rtol(ok_, fmt) * np.abs(os_.astype(np.float64)), 2.0 ** -149)
    assert np.all(np.abs(gs.astype(np.float64) - os_) <= tol)
    if not expand:
        assert np.array_equal(gs, os_)
    diff, maxd = compare_codes(gq, oq)
    assert maxd <= 1
    assert diff.sum() <= max(1, FLIP_FRACTION * diff.size), int(diff.sum())


@pytest.mark.parametrize("gr", [1, 128])
@pytest.mark.parametrize("fmt", [E4M3, E5M2, E5M2_FULL])
@pytest.mark.parametrize("rows,cols", [(256, 640), (100, 650)])
def test_group_dequantize_vs_oracle(orc, gr, fmt, rows, cols):
    """cols = 650: rows that are not a multiple of 16 wide (the ragged kernel),
    strided buffers, a partial 128x128 block."""
    rng = np.random.default_rng(30 + gr + fmt)
    top = 0x7E if fmt == E4M3 else 0x7B
    q = rng.integers(0, top + 1, (rows, cols)).astype(np.uint8) | \
        rng.choice([0, 0x80], (rows, cols)).astype(np.uint8)
    nbr, nbc = -(-rows // gr), -(-cols // 128)
    k = rng.uniform(1.0, 16.0, (nbr, nbc)).astype(np.float32)
    k[:, ::2] = 1.0                  # k = 1 groups beside expanded ones (the exact decode)
    s = np.exp(rng.uniform(-25, 0, (nbr, nbc))).astype(np.float32)
    ref = orc.group_dequantize(q, s, k, gr, 128, fmt)
    ld = -(-cols // 16) * 16           # row strides that are multiples of 16 bytes
    qd = torch.zeros((rows, ld), dtype=torch.uint8, device="cuda")
    qd[:, :cols] = torch.from_numpy(q).cuda()
    qd = qd[:, :cols]
    out = torch.zeros((rows, ld), dtype=torch.float32, device="cuda")[:, :cols]
    coat.coat_group_dequantize(qd, torch.from_numpy(s).cuda(), torch.from_numpy(k).cuda(), gr,
                               128, fmt, out)
    got = out.cpu().numpy().astype(np.float64)
    # x = s * 2^(log2|q| / k): FP32 exponent arithmetic and MUFU ex2 give a few
    # 1e-7 relative (the argument reaches |log2 q| <= 16 at k = 1)
    assert np.all(np.sign(got) == np.sign(ref))
    assert rel_err(got[ref != 0], ref[ref != 0]).max() < 2e-6
    # k = 1: s * value(q) with one rounding, equal to the oracle's exact product rounded
    k1 = np.repeat(np.repeat(k == 1.0, gr, axis=0), 128, axis=1)[:rows, :cols]
    assert np.array_equal(got[k1], ref[k1].astype(np.float32).astype(np.float64))
    outb = torch.zeros((rows, ld), dtype=torch.bfloat16, device="cuda")[:, :cols]
    coat.coat_group_dequantize(qd, torch.from_numpy(s).cuda(), torch.from_numpy(k).cuda(), gr,
                               128, fmt, outb)
    gb = outb.float().cpu().numpy()
    assert np.array_equal(gb, torch.from_numpy(got.astype(np.float32)).bfloat16().float().numpy())
