"""The seeded generators: deterministic, independent of block size, and of
the stated distributions."""
import numpy as np
import pytest

from bitlinear_b1_fwd_b200 import synth


def test_splitmix64_reference_values():
    # splitmix64 seeded with 0: first outputs of the published generator
    z = synth.splitmix64(0, 0, 3)
    assert [hex(int(v)) for v in z] == ["0xe220a8397b1dcdaf", "0x6e789e6aa1b965f4", "0x6c45d188009454f"]


def test_deterministic_and_blockwise():
    a = synth.normal_f32(123, (1000, 37), 0.5)
    b = synth.normal_f32(123, (1000, 37), 0.5)
    assert np.array_equal(a, b)
    old = synth._BLOCK
    try:
        synth._BLOCK = 1000
        c = synth.normal_f32(123, (1000, 37), 0.5)
    finally:
        synth._BLOCK = old
    assert np.array_equal(a, c)
    assert not np.array_equal(a, synth.normal_f32(124, (1000, 37), 0.5))


def test_moments():
    x = synth.normal_f32(7, (1 << 20,), 0.02).astype(np.float64)
    assert x.mean() == pytest.approx(0.0, abs=1e-4)
    assert x.std() == pytest.approx(0.02, rel=5e-3)
    u = synth.uniform(9, 1 << 20)
    assert u.min() >= 0.0 and u.max() < 1.0 and u.mean() == pytest.approx(0.5, abs=2e-3)


def test_outlier_patterns():
    W, x = synth.tiny_inputs()
    assert W.shape == (512, 256) and x.shape == (8, 256)
    base = synth.normal_f32(2001, (8, 256))
    ratio = np.isclose(x, base * 20).mean()
    assert 0.002 < ratio < 0.03
    xc = synth.channel_outliers(base, 3003, 16, 30.0)
    changed = np.nonzero((xc != base).any(axis=0))[0]
    assert len(changed) == 16
