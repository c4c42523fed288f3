"""Pins for the oracle's pre-norm: LayerNorm of each token (fixed-order fp64
mean and variance, bf16 output) followed by per-token absmax INT8 (CPU only).

The pins: exact rational arithmetic on integer tokens (the mean and variance
of integers are exact fractions, the normalized values then follow from one
high-precision square root), the shift invariance that holds exactly for
integer tokens, a constant token (normalized values 0, y = b), an independent
fp64 computation in numpy's own order, and the composition with the pinned
activation quantization."""
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

from bitlinear_b1_fwd_b200 import synth


def _bf16_rne(v: float) -> np.uint16:
    """fp64 -> fp32 (RNE) -> bf16 (RNE), written here with numpy, not the oracle."""
    u = int(np.float32(v).view(np.uint32))
    if (u & 0x7FFFFFFF) > 0x7F800000:
        return np.uint16((u >> 16) | 0x40)
    u += 0x7FFF + ((u >> 16) & 1)
    return np.uint16((u >> 16) & 0xFFFF)


def _bf16_to_f32(h) -> np.ndarray:
    return (np.asarray(h, np.uint32) << 16).view(np.float32)


def _exact_layernorm(row, eps):
    """LayerNorm of an integer row with g = 1, b = 0 in exact rational
    arithmetic (mean, variance) and a 50-digit square root."""
    K = len(row)
    mu = Fraction(sum(int(v) for v in row), K)
    var = sum((Fraction(int(v)) - mu) ** 2 for v in row) / K
    getcontext().prec = 50
    d = var + Fraction(np.float32(eps).item())
    sq = (Decimal(d.numerator) / Decimal(d.denominator)).sqrt()
    return [float((Decimal((Fraction(int(v)) - mu).numerator) / Decimal((Fraction(int(v)) - mu).denominator)) / sq)
            for v in row]


@pytest.mark.parametrize("K", [8, 255, 256, 300, 1000])
def test_integer_tokens_against_exact_arithmetic(orc, K):
    """Integer tokens: the fp64 mean and variance are within a few fp64 ulps
    of the exact fractions, so every bf16 output equals the exact value
    rounded to fp32 then bf16 (a value within 1e-12 relative of a rounding
    boundary would be the only exception; none occurs here)."""
    rng = np.random.default_rng(K)
    x = rng.integers(-50, 51, size=(2, K)).astype(np.float32)
    g = np.ones(K, np.float32)
    b = np.zeros(K, np.float32)
    y = orc.layernorm(x, g, b, eps=1e-5)
    for m in range(2):
        want = np.array([_bf16_rne(v) for v in _exact_layernorm(x[m], 1e-5)], np.uint16)
        assert np.array_equal(y[m], want)


def test_hand_token():
    """x = 1..8, g = 1, b = 0: mu = 4.5, var = 5.25, so y = (k - 4.5) / sqrt(5.25 + 1e-5)."""
    import oracle
    oracle.build()
    x = np.arange(1, 9, dtype=np.float32).reshape(1, 8)
    y = oracle.layernorm(x, np.ones(8, np.float32), np.zeros(8, np.float32))
    want = [(k - 4.5) / np.sqrt(5.25 + float(np.float32(1e-5))) for k in range(1, 9)]
    assert np.array_equal(y[0], np.array([_bf16_rne(v) for v in want], np.uint16))
    assert _bf16_to_f32(y[0])[0] == np.float32(-1.53125)


def test_shift_invariance_integer_tokens(orc):
    """Adding an integer c to an integer token shifts the exact fp64 sums by
    K c and the mean by c, so x - mu and every output are unchanged."""
    rng = np.random.default_rng(5)
    x = rng.integers(-100, 101, size=(3, 777)).astype(np.float32)
    g = synth.normal_f32(51, (777,), 1.0)
    b = synth.normal_f32(52, (777,), 0.1)
    y0 = orc.layernorm(x, g, b)
    y1 = orc.layernorm(x + np.float32(1000.0), g, b)
    assert np.array_equal(y0, y1)


def test_constant_token_gives_bias(orc):
    """A constant token has x - mu = 0 exactly (the sum of K copies is exact),
    so y = b rounded to bf16, and its codes are those of b."""
    K = 1000
    x = np.full((1, K), 0.375, np.float32)
    g = synth.normal_f32(53, (K,), 1.0)
    b = synth.normal_f32(54, (K,), 0.5)
    y, xq, s = orc.layernorm_quant(x, g, b)
    assert np.array_equal(y[0], np.array([_bf16_rne(float(v)) for v in b], np.uint16))
    xq_b, s_b = orc.act_quant(y)
    assert np.array_equal(xq, xq_b) and np.array_equal(s, s_b)


def test_against_numpy_fp64(orc):
    """Random bf16 tokens, weights and biases: numpy's fp64 LayerNorm in its own
    summation order agrees on every bf16 output up to one ulp, and exactly on
    almost all of them (the orders differ only in the last fp64 bits)."""
    M, K = 16, 3200
    x = synth.to_bf16_bits(synth.normal_f32(55, (M, K)))
    g = synth.normal_f32(56, (K,), 1.0)
    b = synth.normal_f32(57, (K,), 0.1)
    y = orc.layernorm(x, g, b)
    xf = _bf16_to_f32(x).astype(np.float64)
    mu = xf.mean(axis=1, keepdims=True)
    var = ((xf - mu) ** 2).mean(axis=1, keepdims=True)
    ref = ((xf - mu) / np.sqrt(var + float(np.float32(1e-5)))) * g.astype(np.float64) + b.astype(np.float64)
    want = np.array([[_bf16_rne(v) for v in row] for row in ref], np.uint16)
    diff = np.abs(y.astype(np.int32) - want.astype(np.int32))
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.999


def test_unit_mean_and_variance(orc):
    """With g = 1, b = 0 the outputs have mean ~0 and variance ~1 (to bf16 precision)."""
    x = synth.normal_f32(58, (8, 4096), 3.0) + np.float32(2.0)
    y = _bf16_to_f32(orc.layernorm(x, np.ones(4096, np.float32), np.zeros(4096, np.float32))).astype(np.float64)
    assert np.all(np.abs(y.mean(axis=1)) < 1e-3)
    assert np.all(np.abs(y.var(axis=1) - 1.0) < 1e-2)


def test_quantization_is_the_pinned_step(orc):
    """x_q and the scales are exactly the activation quantization of the bf16 output."""
    x = synth.normal_f32(59, (5, 1000))
    g = synth.normal_f32(60, (1000,), 1.0)
    b = synth.normal_f32(61, (1000,), 0.1)
    y, xq, s = orc.layernorm_quant(x, g, b)
    xq2, s2 = orc.act_quant(y)
    assert np.array_equal(xq, xq2) and np.array_equal(s, s2)
    assert np.abs(xq).max() == 127
