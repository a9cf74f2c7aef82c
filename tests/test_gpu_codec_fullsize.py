"""Codec parity at the benchmark's full sizes, in the launch configuration the
codec benchmark times: activations 8192 x 4096 in 1x128 groups and weights
4096 x 11008 in 128x128 blocks, bf16, E4M3, expansion off and on, one launch
over the whole tensor.  The oracle checks sampled rows (1x128) and sampled
block rows (128x128), their inputs regenerated on the host from the same
counters; the dequantiser runs over a full-size tensor of generated codes and
is checked on sampled rows."""
import numpy as np
import pytest
import torch

import fp8_optimizer_state_b200 as coat
import synth
from tests.parity import rel_err
from tests.test_gpu_codec import _check_quant

pytestmark = pytest.mark.gpu
E4M3 = 0


@pytest.mark.parametrize("expand", [False, True])
def test_activations_1x128_full_size_sampled_rows(orc, expand):
    R, C = 8192, 4096
    x = torch.empty(R, C, dtype=torch.bfloat16, device="cuda")
    synth.device_activations(x.view(torch.int16).view(-1), 0, 0)
    q = torch.empty(R, C, dtype=torch.uint8, device="cuda")
    s = torch.empty(R, C // 128, dtype=torch.float32, device="cuda")
    k = torch.empty(R, C // 128, dtype=torch.float32, device="cuda")
    coat.coat_group_quantize(x, 1, 128, expand, E4M3, q, s, k)
    torch.cuda.synchronize()
    rows = sorted(set([0, 1, 2, 4095, 4096, R - 1] +
                      list(np.random.default_rng(60).integers(0, R, 10))))
    xh = np.stack([synth.bf16_bits_to_f32(synth.activations_bits(0, 0, r * C, C)) for r in rows])
    oq, os_, ok_ = orc.group_quantize(xh.astype(np.float64), 1, 128, expand, E4M3)
    ri = torch.tensor(rows, device="cuda")
    _check_quant(q[ri].cpu().numpy(), s[ri].cpu().numpy(), k[ri].cpu().numpy(), oq, os_, ok_,
                 E4M3)
    if not expand:
        assert np.array_equal(s[ri].cpu().numpy(), os_)


@pytest.mark.parametrize("expand", [False, True])
def test_weights_128x128_full_size_sampled_block_rows(orc, expand):
    R, C = 4096, 11008
    x = torch.empty(R, C, dtype=torch.bfloat16, device="cuda")
    synth.device_weight(x.view(torch.int16).view(-1), 0, 1)
    nbc = C // 128
    q = torch.empty(R, C, dtype=torch.uint8, device="cuda")
    s = torch.empty(R // 128, nbc, dtype=torch.float32, device="cuda")
    k = torch.empty(R // 128, nbc, dtype=torch.float32, device="cuda")
    coat.coat_group_quantize(x, 128, 128, expand, E4M3, q, s, k)
    torch.cuda.synchronize()
    for br in (0, 17, R // 128 - 1):
        r0 = br * 128
        xh = synth.bf16_bits_to_f32(synth.weight_bits(0, 1, r0 * C, 128 * C)).reshape(128, C)
        oq, os_, ok_ = orc.group_quantize(xh.astype(np.float64), 128, 128, expand, E4M3)
        _check_quant(q[r0:r0 + 128].cpu().numpy(), s[br:br + 1].cpu().numpy(),
                     k[br:br + 1].cpu().numpy(), oq, os_, ok_, E4M3)


def test_dequantize_full_size_sampled_rows(orc):
    """Generated codes (E4M3 over its range, random signs) with per-group k in
    [1.5, 2.2) and root scales; every group of the first rows forced to k = 1
    (the exact path), which must then equal the oracle bit for bit."""
    R, C = 8192, 4096
    ng = C // 128
    q = torch.empty(R, C, dtype=torch.uint8, device="cuda")
    synth.device_state_codes(q.view(-1), 3, 0, 1, E4M3, True)
    km, sm, kv, sv = (torch.empty(R * ng, dtype=torch.float32, device="cuda") for _ in range(4))
    synth.device_state_groups(km, sm, kv, sv, 3, 0, 1)
    k = km.view(R, ng).clone()
    k[:8] = 1.0
    s = sm.view(R, ng)
    out = torch.empty(R, C, dtype=torch.float32, device="cuda")
    coat.coat_group_dequantize(q, s, k, 1, 128, E4M3, out)
    torch.cuda.synchronize()
    rows = [0, 3, 7, 8, 100, 4097, R - 1]
    for r in rows:
        qh = synth.state_codes(3, 0, 1, r * C, C, E4M3, True).reshape(1, C)
        kh, shh, _, _ = synth.state_groups(3, 0, 1, r * ng, ng)
        kh = kh.reshape(1, ng).copy()
        if r < 8:
            kh[:] = 1.0
        ref = orc.group_dequantize(qh, shh.reshape(1, ng), kh, 1, 128, E4M3)
        got = out[r:r + 1].cpu().numpy().astype(np.float64)
        assert np.all(np.sign(got) == np.sign(ref))
        nz = ref != 0
        if r < 8:
            assert np.array_equal(got, ref.astype(np.float32).astype(np.float64)), r
        else:
            assert rel_err(got[nz], ref[nz]).max() < 2e-6, r
