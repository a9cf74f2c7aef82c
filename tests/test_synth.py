"""The seeded input generator: determinism and the workload distributions.
(The device generator's bit-equality with this host one is checked in
test_gpu_synth.py.)"""
import numpy as np

import synth


def test_deterministic_and_stream_separated():
    a = synth.master(0, 3, 1000, 5000)
    b = synth.master(0, 3, 1000, 5000)
    assert np.array_equal(a, b)
    # a window is a slice of a longer draw (counter = element index)
    c = synth.master(0, 3, 0, 6000)
    assert np.array_equal(a, c[1000:])
    assert not np.array_equal(a, synth.master(1, 3, 1000, 5000))
    assert not np.array_equal(a, synth.master(0, 4, 1000, 5000))
    g1 = synth.grad_bits(0, 3, 1, 0, 4096)
    g2 = synth.grad_bits(0, 3, 2, 0, 4096)
    assert not np.array_equal(g1, g2)


def test_philox_words_look_uniform():
    w = np.concatenate(synth.philox4x32_10(np.arange(200000, dtype=np.uint32), 0, 7, 0, 123, 9))
    top = (w >> np.uint32(28)).astype(np.int64)
    counts = np.bincount(top, minlength=16)
    expect = w.size / 16
    chi2 = float(((counts - expect) ** 2 / expect).sum())
    assert chi2 < 50.0           # 15 dof; p ~ 1e-5
    assert abs(w.astype(np.float64).mean() / 2 ** 32 - 0.5) < 0.005


def test_normal_and_master_moments():
    x = synth.master(0, 0, 0, 400000).astype(np.float64) / synth.MASTER_SIGMA
    assert abs(x.mean()) < 0.01
    assert abs(x.std() - 1.0) < 0.01
    assert np.abs(x).max() <= 2 * np.sqrt(3.0) + 1e-9


def test_state_group_ratios():
    n = 128 * 500
    m = synth.m_warm(0, 0, 0, n).astype(np.float64).reshape(-1, 128)
    v = synth.v_warm(0, 0, 0, n).astype(np.float64).reshape(-1, 128)
    sg = synth.group_scale(0, 0, 0, 500).astype(np.float64)
    am = np.abs(m)
    rm = am.max(1) / am.min(1)
    rv = v.max(1) / v.min(1)
    # page: first-moment groups max/min ~1000, second-moment ~10
    assert 300 < np.median(rm) <= 1000.0 and rm.max() <= 1000.0 * 1.0001
    assert 4 < np.median(rv) <= 10.0 and rv.max() <= 10.0 * 1.0001
    assert np.all(am.max(1) <= sg * 1.000001) and np.all(v.max(1) <= sg ** 2 * 1.000001)
    assert 0.4 < (m < 0).mean() < 0.6
    lg = np.log10(sg)
    assert lg.min() >= -5.0001 and lg.max() <= -1.9999


def test_grad_is_bf16_of_scaled_normal():
    n = 128 * 64
    g = synth.bf16_bits_to_f32(synth.grad_bits(0, 1, 1, 0, n)).astype(np.float64).reshape(-1, 128)
    sg = synth.group_scale(0, 1, 0, 64).astype(np.float64)
    z = g / sg[:, None]
    assert abs(z.std() - 1.0) < 0.05
    # a window starting mid-group uses the right group scales
    w = synth.grad_bits(0, 1, 1, 200, 300)
    assert np.array_equal(w, synth.grad_bits(0, 1, 1, 0, n)[200:500])


def test_activation_outliers():
    a = synth.bf16_bits_to_f32(synth.activations_bits(0, 0, 0, 1 << 20)).astype(np.float64)
    frac = (np.abs(a) > 4.0).mean()
    assert 0.0006 < frac < 0.0014   # ~0.1% outliers x100 (|z| <= 3.47 otherwise)
