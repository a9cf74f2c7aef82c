"""GPU parity of the FP8 SwiGLU layer (coat_swiglu_fp8_forward / _backward)
against the oracle, through the C ABI.

Inputs: synthetic activations (unit scale, 0.1% outliers at 100x) quantised
per 1x128 group by the oracle's codec, with or without expansion, so both
sides start from the same FP8 gate / up.

Forward: k within 1e-5 and the root scale within the k-derived bound (the
codec's rules); codes within one step, and every differing code is a tie: the
exact expanded value lies within 2e-6 (plus what the k difference moves it)
of the midpoint between the two codes.  Ties are common here, unlike in the
optimizer step: elements of a group that share a gate value have
h_i / h_max = u_i / u_max, a ratio of two FP8 values, which often lands
exactly on a rounding midpoint; each side's FP32 roundings of h_i and h_max
then break the tie their own way (about 1e-4 of the elements, measured with
exact FP32 arithmetic as well).  At most 1e-3 of the codes may differ.

Backward: bf16 gradients within one bf16 ulp of the oracle's, plus a term for
cancellation in 1 + g (1 - sigmoid(g)), with at most 2e-3 of the elements off
by that ulp."""
import numpy as np
import pytest
import torch

import fp8_optimizer_state_b200 as coat
import oracle
import synth
from tests.parity import K_RTOL, code_ordinal, rel_err, scale_rtol

pytestmark = pytest.mark.gpu
E4M3, E5M2, E5M2_FULL = 0, 1, 2
ULP_FRACTION = 2e-3     # device sigmoid / product error (~1e-6 rel) against the bf16 ulp (2^-8)


def make_inputs(orc, rows, cols, fmt, expand_in, seed):
    """expand_in: one flag for both inputs, or a (gate, up) pair."""
    flags = expand_in if isinstance(expand_in, tuple) else (expand_in, expand_in)
    acts = []
    for t in (0, 1):
        bits = synth.activations_bits(seed, t, 0, rows * cols).reshape(rows, cols)
        x = synth.bf16_bits_to_f32(bits).astype(np.float64)
        acts.append(orc.group_quantize(x, 1, 128, flags[t], fmt))
    return acts


def to_dev(a):
    q, s, k = a
    return (torch.from_numpy(np.ascontiguousarray(q)).cuda(),
            torch.from_numpy(np.ascontiguousarray(s)).cuda(),
            torch.from_numpy(np.ascontiguousarray(k)).cuda())


def empty_act(rows, cols):
    ng = -(-cols // 128)
    return (torch.zeros((rows, cols), dtype=torch.uint8, device="cuda"),
            torch.zeros((rows, ng), dtype=torch.float32, device="cuda"),
            torch.zeros((rows, ng), dtype=torch.float32, device="cuda"))


def host(a):
    torch.cuda.synchronize()
    return tuple(t.cpu().numpy() for t in a)


TIE_RTOL = 2e-6         # FP32 roundings of h on both sides (~4 each) and the approximate sigmoid
FLIP_LIMIT = 1e-3


def exact_h(orc, gate, up, fmt):
    """h = silu(g) u in double from the dequantised FP8 inputs (the sigmoid flushed
    below 2^-126 as in the oracle)."""
    g = orc.group_dequantize(*gate, 1, 128, fmt)
    u = orc.group_dequantize(*up, 1, 128, fmt)
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-g))
    s = np.where(s < 2.0 ** -126, 0.0, s)
    return g * s * u


def check_act(tag, fmt, dev, orc_out, h):
    """Forward comparison over a [rows, cols] 1x128 tensor (module docstring).
    h: the exact activation values, for the tie test."""
    qd, sd, kd = (np.asarray(a) for a in dev)
    qo, so, ko = (np.asarray(a) for a in orc_out)
    assert rel_err(kd, ko).max() <= K_RTOL, "%s: k rel err %.3g" % (tag, rel_err(kd, ko).max())
    se, tol = rel_err(sd, so), scale_rtol(ko, fmt)
    assert np.all(se <= tol), "%s: scale rel err %.3g" % (tag, se.max())
    step = np.abs(code_ordinal(qd) - code_ordinal(qo))
    assert step.max() <= 1, "%s: a code differs by %d steps" % (tag, step.max())
    flips = np.argwhere(step != 0)
    table = np.abs(oracle.fp8_decode_table(fmt))
    fmax = table[0x7E if fmt == E4M3 else 0x7B]
    for r, c in flips:
        j = c // 128
        grp = np.abs(h[r, j * 128:(j + 1) * 128])
        M = grp[np.isfinite(grp)].max()
        ratio = abs(h[r, c]) / M
        y = fmax * ratio ** float(ko[r, j])
        mid = 0.5 * (table[qd[r, c] & 0x7F] + table[qo[r, c] & 0x7F])
        allow = TIE_RTOL + abs(np.log(ratio)) * abs(float(kd[r, j]) - float(ko[r, j]))
        assert abs(y - mid) <= allow * mid, "%s: code flip at (%d, %d) is not a tie: y=%.9g, " \
            "midpoint %.9g" % (tag, r, c, y, mid)
    assert len(flips) <= max(2, FLIP_LIMIT * qo.size), "%s: %d flips" % (tag, len(flips))
    return len(flips)


def bf16_f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16) \
        .to(torch.float64).numpy()


def ulp_bf16(x):
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def check_grad(tag, dev_bits, orc_bits, terms):
    """dev within one bf16 ulp of the oracle's value plus 4e-6 of `terms` (the
    size of the summands, for cancellation); off-by-one-ulp elements limited."""
    d, o = bf16_f64(dev_bits), bf16_f64(orc_bits)
    assert np.array_equal(np.isnan(d), np.isnan(o)), tag + ": NaN positions"
    m = ~np.isnan(o)
    err = np.abs(d[m] - o[m])
    tol = ulp_bf16(np.maximum(np.abs(d[m]), np.abs(o[m]))) + 4e-6 * terms[m]
    assert np.all(err <= tol), "%s: %d elements beyond one ulp (worst %.3g vs %.3g)" % (
        tag, int((err > tol).sum()), float(err.max()), float(tol[np.argmax(err - tol)]))
    nd = int((err > 0).sum())
    assert nd <= max(2, ULP_FRACTION * err.size), "%s: %d of %d differ" % (tag, nd, err.size)
    return nd


def forward_case(orc, rows, cols, fmt, expand_in, expand_out, seed=1):
    gate, up = make_inputs(orc, rows, cols, fmt, expand_in, seed)
    out = empty_act(rows, cols)
    coat.coat_swiglu_fp8_forward(to_dev(gate), to_dev(up), fmt, expand_out, out)
    want = orc.swiglu_fp8_forward(gate, up, fmt, expand_out)
    return check_act("swiglu fwd %dx%d" % (rows, cols), fmt, host(out), want,
                     exact_h(orc, gate, up, fmt))


@pytest.mark.parametrize("rows,cols,fmt,expand_in,expand_out", [
    (64, 1024, E4M3, False, False),       # the usual case: no expansion anywhere
    (33, 11008, E4M3, False, False),      # a Llama-2-7B MLP width (86 groups), ragged quads
    (40, 1024, E4M3, True, True),         # expanded inputs (table decode) and output
    (24, 1024, E4M3, (False, True), False),   # k = 1 gate beside expanded up in one warp
    (17, 304, E5M2, False, False),        # E5M2; a partial last group of 48
    (9, 304, E5M2_FULL, False, True),
    (5, 16, E4M3, False, True),           # one partial group per row
    (1, 128, E4M3, False, False),
])
def test_forward_vs_oracle(orc, rows, cols, fmt, expand_in, expand_out):
    flips = forward_case(orc, rows, cols, fmt, expand_in, expand_out)
    print("flips", flips)


def test_forward_fused_gate_up_buffer_and_strided_output(orc):
    """gate and up as the two halves of one [rows, 2F] buffer (the fused
    up/gate projection's output), the result into a view of a wider buffer."""
    rows, F, fmt = 24, 640, E4M3
    gate, up = make_inputs(orc, rows, F, fmt, False, 4)
    qb = torch.from_numpy(np.concatenate([gate[0], up[0]], axis=1)).cuda()
    sb = torch.from_numpy(np.concatenate([gate[1], up[1]], axis=1)).cuda()
    kb = torch.from_numpy(np.concatenate([gate[2], up[2]], axis=1)).cuda()
    g5, ng = F // 128, F // 128
    gd = (qb[:, :F], sb[:, :g5], kb[:, :g5])
    ud = (qb[:, F:], sb[:, g5:], kb[:, g5:])
    wide = (torch.zeros((rows, F + 32), dtype=torch.uint8, device="cuda"),
            torch.zeros((rows, ng + 3), dtype=torch.float32, device="cuda"),
            torch.zeros((rows, ng + 3), dtype=torch.float32, device="cuda"))
    out = (wide[0][:, :F], wide[1][:, :ng], wide[2][:, :ng])
    coat.coat_swiglu_fp8_forward(gd, ud, fmt, False, out)
    want = orc.swiglu_fp8_forward(gate, up, fmt, False)
    check_act("fused", fmt, host(out), want, exact_h(orc, gate, up, fmt))
    hw = host(wide)
    assert not hw[0][:, F:].any() and not hw[1][:, ng:].any()   # nothing written past the view


def test_forward_special_values(orc):
    """NaN codes in the inputs: their outputs are NaN codes, and a group's
    other elements follow the oracle (the maximum ignores NaN); a group whose
    every value is NaN is all zero codes with k = 1, scale 1 (the codec's
    rule)."""
    rows, cols, fmt = 4, 512, E4M3
    gate, up = make_inputs(orc, rows, cols, fmt, False, 5)
    gate[0][0, 3] = 0x7F
    up[0][1, 200] = 0xFF
    gate[0][2, 256:384] = 0x7F                     # a whole group of NaN
    out = empty_act(rows, cols)
    coat.coat_swiglu_fp8_forward(to_dev(gate), to_dev(up), fmt, False, out)
    qd, sd, kd = host(out)
    qo, so, ko = orc.swiglu_fp8_forward(gate, up, fmt, False)
    nan = np.zeros((rows, cols), bool)
    nan[0, 3] = nan[1, 200] = True
    assert not qd[2, 256:384].any() and sd[2, 2] == 1.0 and kd[2, 2] == 1.0
    assert np.all((qd[nan] & 0x7F) == 0x7F) and np.all((qo[nan] & 0x7F) == 0x7F)
    qd2, qo2 = qd.copy(), qo.copy()
    qd2[nan] = qo2[nan] = 0
    check_act("special", fmt, (qd2, sd, kd), (qo2, so, ko), exact_h(orc, gate, up, fmt))


def grad_terms(orc, gate, up, dh, fmt):
    """Magnitudes of the products that form dgate and dup (for cancellation)."""
    g = orc.group_dequantize(*gate, 1, 128, fmt)
    u = orc.group_dequantize(*up, 1, 128, fmt)
    d = bf16_f64(dh)
    s = 1.0 / (1.0 + np.exp(-np.clip(g, -700, 700)))
    return np.abs(d * u * s) * (1.0 + np.abs(g) * (1.0 - s)), np.abs(d * g * s)


def backward_case(orc, rows, cols, fmt, expand_in, seed=2):
    gate, up = make_inputs(orc, rows, cols, fmt, expand_in, seed)
    dh = synth.grad_bits(seed, 5, 1, 0, rows * cols).reshape(rows, cols)
    dg = torch.zeros((rows, cols), dtype=torch.int16, device="cuda")
    du = torch.zeros((rows, cols), dtype=torch.int16, device="cuda")
    coat.coat_swiglu_fp8_backward(torch.from_numpy(dh.view(np.int16)).cuda(), to_dev(gate),
                                  to_dev(up), fmt, dg, du)
    og, ou = orc.swiglu_fp8_backward(dh, gate, up, fmt)
    torch.cuda.synchronize()
    terms_g, terms_u = grad_terms(orc, gate, up, dh, fmt)
    n1 = check_grad("dgate", dg.cpu().numpy().view(np.uint16), og, terms_g)
    n2 = check_grad("dup", du.cpu().numpy().view(np.uint16), ou, terms_u)
    return n1, n2


@pytest.mark.parametrize("rows,cols,fmt,expand_in", [
    (64, 1024, E4M3, False),
    (33, 11008, E4M3, False),
    (40, 1024, E4M3, True),
    (24, 1024, E4M3, (False, True)),
    (17, 304, E5M2, False),
    (3, 16, E4M3, False),
])
def test_backward_vs_oracle(orc, rows, cols, fmt, expand_in):
    print("ulp differences", backward_case(orc, rows, cols, fmt, expand_in))


def test_backward_strided_views(orc):
    """The forward's fused [rows, 2F] input buffer read in place; gradients
    written into the two halves of one [rows, 2F] bf16 buffer."""
    rows, F, fmt = 12, 384, E4M3
    gate, up = make_inputs(orc, rows, F, fmt, False, 6)
    qb = torch.from_numpy(np.concatenate([gate[0], up[0]], axis=1)).cuda()
    sb = torch.from_numpy(np.concatenate([gate[1], up[1]], axis=1)).cuda()
    kb = torch.from_numpy(np.concatenate([gate[2], up[2]], axis=1)).cuda()
    g5 = F // 128
    dh = synth.grad_bits(6, 5, 1, 0, rows * F).reshape(rows, F)
    grads = torch.zeros((rows, 2 * F), dtype=torch.int16, device="cuda")
    coat.coat_swiglu_fp8_backward(torch.from_numpy(dh.view(np.int16)).cuda(),
                                  (qb[:, :F], sb[:, :g5], kb[:, :g5]),
                                  (qb[:, F:], sb[:, g5:], kb[:, g5:]), fmt, grads[:, :F],
                                  grads[:, F:])
    og, ou = orc.swiglu_fp8_backward(dh, gate, up, fmt)
    gb = grads.cpu().numpy().view(np.uint16)
    terms_g, terms_u = grad_terms(orc, gate, up, dh, fmt)
    check_grad("dgate strided", np.ascontiguousarray(gb[:, :F]), og, terms_g)
    check_grad("dup strided", np.ascontiguousarray(gb[:, F:]), ou, terms_u)


def test_layer_output_feeds_the_next_fp8_layer(orc):
    """The precision flow: the forward's FP8 output is the next layer's FP8
    input as it stands (here a second SwiGLU as the stand-in consumer), and
    the two-layer chain matches the oracle's chain."""
    rows, cols, fmt = 16, 512, E4M3
    gate, up = make_inputs(orc, rows, cols, fmt, False, 7)
    out1 = empty_act(rows, cols)
    coat.coat_swiglu_fp8_forward(to_dev(gate), to_dev(up), fmt, False, out1)
    o1 = orc.swiglu_fp8_forward(gate, up, fmt, False)
    h1 = host(out1)
    check_act("layer 1", fmt, h1, o1, exact_h(orc, gate, up, fmt))
    # second layer: gate = layer-1 output (each side's own), up = the same up
    out2 = empty_act(rows, cols)
    coat.coat_swiglu_fp8_forward(out1, to_dev(up), fmt, False, out2)
    # compare the rows whose layer-1 codes agree (a flipped code is a different
    # input; the scales differ only within their tolerance, ~1e-7 here, which
    # moves h by about as much and stays inside the tie bound)
    same = np.all(h1[0] == o1[0], axis=1)
    o2 = orc.swiglu_fp8_forward(o1, up, fmt, False)
    h2 = host(out2)
    assert same.sum() >= rows // 2
    check_act("layer 2", fmt, tuple(a[same] for a in h2), tuple(a[same] for a in o2),
              exact_h(orc, o1, up, fmt)[same])


def test_zero_sizes_and_cols_not_multiple_of_16():
    z = empty_act(0, 128)
    coat.coat_swiglu_fp8_forward(z, z, E4M3, False, z)
    a = empty_act(2, 24)
    with pytest.raises(coat.CoatError):
        coat.coat_swiglu_fp8_forward(a, a, E4M3, False, a)


def test_full_size_sampled_rows(orc):
    """The benchmark's shape and launch configuration: 8192 tokens x 11008,
    gate and up the halves of one [T, 2F] E4M3 tensor, gradients into the
    halves of one [T, 2F] bf16 buffer.  Inputs drawn by the seeded generator
    on the device (codes over the format's range, per-group root scales times
    2^10, k = 1); the oracle checks sampled token rows, regenerated on the host
    from the same counters."""
    T, F, fmt = 8192, 11008, E4M3
    ng = F // 128
    xq = torch.empty(T, 2 * F, dtype=torch.uint8, device="cuda")
    xs = torch.empty(T, 2 * ng, dtype=torch.float32, device="cuda")
    xk = torch.ones(T, 2 * ng, dtype=torch.float32, device="cuda")
    tmp_q = torch.empty(T, F, dtype=torch.uint8, device="cuda")
    tmp = [torch.empty(T * ng, dtype=torch.float32, device="cuda") for _ in range(4)]
    for t, (c0, g0) in enumerate(((0, 0), (F, ng))):
        synth.device_state_codes(tmp_q, 8, t, 1, fmt, True)
        synth.device_state_groups(*tmp, 8, t, 1)
        xq[:, c0:c0 + F].copy_(tmp_q)
        xs[:, g0:g0 + ng].copy_(tmp[1].view(T, ng) * 1024.0)
    dh = torch.empty(T, F, dtype=torch.int16, device="cuda")
    synth.device_grad(dh.view(-1), 8, 9, 1)
    gate = (xq[:, :F], xs[:, :ng], xk[:, :ng])
    up = (xq[:, F:], xs[:, ng:], xk[:, ng:])
    out = empty_act(T, F)
    grads = torch.zeros(T, 2 * F, dtype=torch.int16, device="cuda")
    coat.coat_swiglu_fp8_forward(gate, up, fmt, False, out)
    coat.coat_swiglu_fp8_backward(dh, gate, up, fmt, grads[:, :F], grads[:, F:])
    torch.cuda.synchronize()
    rows = [0, 1, 777, 4095, 4096, 6000, T - 2, T - 1]
    for r in rows:
        host_in = []
        for t in (0, 1):
            q = synth.state_codes(8, t, 1, r * F, F, fmt, True).reshape(1, F)
            s = synth.state_groups(8, t, 1, r * ng, ng)[1].reshape(1, ng) * np.float32(1024.0)
            host_in.append((q, s.astype(np.float32), np.ones((1, ng), np.float32)))
        assert np.array_equal(host_in[0][0][0], xq[r, :F].cpu().numpy())
        want = orc.swiglu_fp8_forward(host_in[0], host_in[1], fmt, False)
        got = tuple(a[r:r + 1].cpu().numpy() for a in out)
        check_act("row %d" % r, fmt, got, want, exact_h(orc, host_in[0], host_in[1], fmt))
        d = synth.grad_bits(8, 9, 1, r * F, F).reshape(1, F)
        og, ou = orc.swiglu_fp8_backward(d, host_in[0], host_in[1], fmt)
        tg, tu = grad_terms(orc, host_in[0], host_in[1], d, fmt)
        gb = grads[r:r + 1].cpu().numpy().view(np.uint16)
        check_grad("dgate row %d" % r, np.ascontiguousarray(gb[:, :F]), og, tg)
        check_grad("dup row %d" % r, np.ascontiguousarray(gb[:, F:]), ou, tu)
