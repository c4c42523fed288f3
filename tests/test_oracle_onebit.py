"""Pins for the oracle's 1-bit variant: alpha, beta and the {-1, +1} codes of
a whole matrix, the 8-weights-per-byte format and the forward with beta as the
weight factor (CPU only).

The pins: the pages' five-weight example (golden file), exact rational
arithmetic on integer matrices, the tie rule on a hand-made matrix, numpy's
own fp64 sums, a hand-packed byte, and brute-force integer products."""
from fractions import Fraction

import numpy as np
import pytest

from conftest import read_golden
from bitlinear_b1_fwd_b200 import synth

B1 = 2


def test_worked_example_b_whole_matrix(orc):
    """The pages' example through the matrix routine: beta = 0.57, alpha =
    -0.03, signs [+1, -1, +1, -1, +1], and the 0.05 weight sent to +beta."""
    g = read_golden("worked_example_b.txt")
    w = np.array([[float(v) for v in g["w"]]], np.float32)
    alpha, beta, codes = orc.binarize_weights(w)
    assert round(float(beta), 2) == float(g["beta"][0])
    assert float(alpha) == pytest.approx(-0.03, abs=1e-6)
    assert codes[0].tolist() == [1, -1, 1, -1, 1]
    i = int(g["onebit_err_idx"][0])
    assert round(abs(float(beta) * codes[0, i] - float(w[0, i])), 2) == float(g["onebit_err"][0])


@pytest.mark.parametrize("shape", [(1, 7), (3, 1000), (5, 8192), (37, 3001)])
def test_alpha_beta_exact_on_integers(orc, shape):
    """Integer weights: every fp64 partial sum is exact, so alpha and beta are
    the exact means rounded once to fp64 and once to fp32."""
    rng = np.random.default_rng(shape[1])
    W = rng.integers(-60, 41, size=shape).astype(np.float32)
    T = W.size
    S = int(W.astype(np.int64).sum())
    A = int(np.abs(W).astype(np.int64).sum())
    alpha, beta, codes = orc.binarize_weights(W)
    assert alpha == np.float32(float(Fraction(S, T)))
    assert beta == np.float32(float(Fraction(A, T)))
    assert orc.signed_sum(W) == float(S)
    # the sign of w - alpha against the exact mean
    mean = Fraction(S, T)
    want = np.array([[1 if Fraction(int(v)) > Fraction(float(alpha)) else -1 for v in row] for row in W], np.int8)
    assert np.array_equal(codes, want)
    # the exact mean and its fp32 rounding agree on every integer weight
    assert all((Fraction(int(v)) > mean) == (float(v) > float(alpha)) for v in W.ravel()[:500])


def test_tie_maps_to_minus_one(orc):
    """A weight equal to alpha is not above it: [1, 2, 3] has alpha = 2."""
    alpha, beta, codes = orc.binarize_weights(np.array([[1.0, 2.0, 3.0]], np.float32))
    assert alpha == np.float32(2.0) and beta == np.float32(2.0)
    assert codes[0].tolist() == [-1, -1, 1]


def test_bf16_weights_alpha_beta_against_numpy(orc):
    """Random bf16 matrices: numpy's fp64 sums (its own order) give the same
    fp32 alpha and beta to within one fp32 ulp."""
    for seed, (N, K) in enumerate([(64, 3200), (300, 1000)]):
        Wf = synth.normal_f32(500 + seed, (N, K), 0.02) + np.float32(0.001)
        W = synth.to_bf16_bits(Wf)
        Wd = (W.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        alpha, beta, codes = orc.binarize_weights(W)
        a_ref = np.float32(Wd.sum() / Wd.size)
        b_ref = np.float32(np.abs(Wd).sum() / Wd.size)
        assert abs(int(alpha.view(np.int32)) - int(a_ref.view(np.int32))) <= 1
        assert abs(int(beta.view(np.int32)) - int(b_ref.view(np.int32))) <= 1
        assert beta == orc.gamma(W)
        # codes: above alpha -> +1, else -1; both signs occur about equally
        assert np.array_equal(codes, np.where(Wd.astype(np.float32) > alpha, 1, -1).astype(np.int8))
        assert abs(float((codes == 1).mean()) - 0.5) < 0.02


def test_pack_hand_byte(orc):
    """Bit i of byte j holds weight 8 j + i (1 for +1); pad bits are 0."""
    codes = np.array([[1, -1, -1, 1, 1, 1, -1, 1, 1]], np.int8)
    p = orc.pack(codes, B1)
    assert p.shape == (1, 16)
    assert p[0, 0] == 0b10111001 and p[0, 1] == 0x01
    assert not p[0, 2:].any()
    assert np.array_equal(orc.unpack(p, 1, 9, B1), codes)
    assert orc.packed_row_bytes(128, B1) == 16 and orc.packed_row_bytes(129, B1) == 32


def test_pack_rejects_zero_and_set_pad_bit(orc):
    with pytest.raises(ValueError):
        orc.pack(np.array([[1, 0, -1]], np.int8), B1)
    p = orc.pack(np.array([[1, -1, -1]], np.int8), B1)
    p[0, 0] |= 0x08  # weight 3 of a row of 3
    with pytest.raises(ValueError):
        orc.unpack(p, 1, 3, B1)


def test_pack_roundtrip_random(orc):
    rng = np.random.default_rng(7)
    for K in (1, 8, 127, 128, 129, 1000):
        codes = np.where(rng.random((5, K)) < 0.5, 1, -1).astype(np.int8)
        p = orc.pack(codes, B1)
        assert np.array_equal(orc.unpack(p, 5, K, B1), codes)
        # the packed bits are numpy's little-endian bit packing of (code > 0)
        want = np.packbits(codes > 0, axis=1, bitorder="little")
        assert np.array_equal(p[:, :want.shape[1]], want)


@pytest.mark.parametrize("xdt", ["f32", "bf16", "i8"])
def test_forward_brute_force(orc, xdt):
    """The forward with 1-bit weights: the INT32 products equal numpy's int64
    products, and the fp32 outputs equal acc * ((beta * s) / 127) in numpy's
    fp32 arithmetic; the product equals 2 * (sum of x_q over the +1 weights)
    minus the sum of x_q."""
    N, K, M = 96, 777, 6
    W = synth.normal_f32(510, (N, K), 0.02)
    alpha, beta, codes = orc.binarize_weights(W)
    packed = orc.pack(codes, B1)
    x = synth.normal_f32(511, (M, K))
    if xdt == "bf16":
        x = synth.to_bf16_bits(x)
    scale = None
    if xdt == "i8":
        x, scale = orc.act_quant(x)
    acc, s = orc.forward(packed, B1, beta, N, K, x, ydt=3, scale=scale)
    xq = x if xdt == "i8" else orc.act_quant(x)[0]
    ref = xq.astype(np.int64) @ codes.astype(np.int64).T
    assert np.array_equal(acc, ref)
    plus = xq.astype(np.int64) @ (codes > 0).astype(np.int64).T
    assert np.array_equal(acc, 2 * plus - xq.astype(np.int64).sum(axis=1, keepdims=True))
    y, _ = orc.forward(packed, B1, beta, N, K, x, ydt=0, scale=scale)
    c = (np.float32(beta) * s.astype(np.float32)) / np.float32(127.0)
    assert np.array_equal(y, ref.astype(np.float32) * c[:, None])
