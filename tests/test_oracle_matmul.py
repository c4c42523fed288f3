"""Pins for the oracle's ternary x INT8 product, dequantization and whole
forward (CPU only): brute force, the add/subtract/skip restatement of the
pages, hand values and the pages' float formulation."""
import numpy as np
import pytest

from conftest import read_golden
from bitlinear_b1_fwd_b200 import synth


def test_brute_force_tiny(orc):
    rng = np.random.default_rng(5)
    for (M, N, K) in [(1, 1, 1), (3, 4, 5), (2, 7, 13), (5, 3, 64)]:
        codes = rng.integers(-1, 2, (N, K), dtype=np.int8)
        xq = rng.integers(-127, 128, (M, K), dtype=np.int8)
        acc = orc.matmul_i32(codes, xq)
        for m in range(M):
            for n in range(N):
                s = 0
                for k in range(K):
                    s += int(codes[n, k]) * int(xq[m, k])
                assert acc[m, n] == s


def test_add_sub_skip_restatement(orc):
    """y_i = sum of x_j over w_ij = +1, minus the sum over w_ij = -1; zeros skipped."""
    rng = np.random.default_rng(6)
    codes = rng.integers(-1, 2, (96, 777), dtype=np.int8)
    xq = rng.integers(-127, 128, (9, 777), dtype=np.int8)
    acc = orc.matmul_i32(codes, xq)
    x64 = xq.astype(np.int64)
    plus = (codes == 1).astype(np.int64)
    minus = (codes == -1).astype(np.int64)
    want = x64 @ plus.T - x64 @ minus.T
    assert np.array_equal(acc.astype(np.int64), want)
    # extreme magnitudes stay exact in int32: all +1 weights against all 127
    big = orc.matmul_i32(np.ones((2, 28672), np.int8), np.full((1, 28672), 127, np.int8))
    assert big.tolist() == [[127 * 28672, 127 * 28672]]
    neg = orc.matmul_i32(-np.ones((1, 28672), np.int8), np.full((1, 28672), 127, np.int8))
    assert neg.tolist() == [[-127 * 28672]]
    # at the largest K the library takes (2^20) the sum still fits INT32 and is exact
    K = 1 << 20
    top = orc.matmul_i32(np.stack([np.ones(K, np.int8), -np.ones(K, np.int8)]), np.full((1, K), 127, np.int8))
    assert top.tolist() == [[127 * K, -127 * K]] and 127 * K < 2 ** 31


def test_parallel_matches_serial(orc):
    rng = np.random.default_rng(8)
    codes = rng.integers(-1, 2, (101, 300), dtype=np.int8)
    xq = rng.integers(-127, 128, (3, 300), dtype=np.int8)
    assert np.array_equal(orc.matmul_i32(codes, xq), orc.matmul_i32(codes, xq, parallel=True))
    W = synth.normal_f32(9, (77, 123), 0.02)
    g = orc.gamma(W)
    assert np.array_equal(orc.ternarize(W, g), orc.ternarize(W, g, parallel=True))


def test_worked_example_forward(orc):
    """Example A's codes against a token of ones: s = 1, x_q = 127 everywhere,
    acc = 127 * (0 - 1 + 1 - 1 + 0) = -127, y = gamma * (-1) = -0.61."""
    g = read_golden("worked_example_a.txt")
    W = np.array([[float(v) for v in g["W"]]], np.float32)
    gamma = orc.gamma(W)
    packed = orc.pack(orc.ternarize(W, gamma), 0)
    x = np.ones((1, 5), np.float32)
    acc, s = orc.forward(packed, 0, gamma, 1, 5, x, ydt=orc.I32)
    assert s.tolist() == [1.0] and acc.tolist() == [[-127]]
    y, _ = orc.forward(packed, 0, gamma, 1, 5, x, ydt=orc.F32)
    assert float(y[0, 0]) == pytest.approx(-float(g["gamma"][0]), abs=1e-6)


@pytest.mark.parametrize("fmt", [0, 1])
def test_forward_vs_pages_float_formula(orc, fmt):
    """The page's BitLinear computes gamma * (x_deq @ W_q^T) with
    x_deq = x_q / 127 * scale in floating point; in fp64 that must agree with
    the oracle's integer path to fp32 rounding."""
    W, x = synth.tiny_inputs()
    gamma = orc.gamma(W)
    codes = orc.ternarize(W, gamma)
    packed = orc.pack(codes, fmt)
    y, s = orc.forward(packed, fmt, gamma, 512, 256, x, ydt=orc.F32)
    xq, s2 = orc.act_quant(x)
    assert np.array_equal(s, s2)
    x_deq = xq.astype(np.float64) / 127.0 * s.astype(np.float64)[:, None]
    ref = float(gamma) * (x_deq @ codes.astype(np.float64).T)
    assert np.allclose(y, ref, rtol=1e-6, atol=1e-12 * np.abs(ref).max())
    # a wrong scale (for example a missing /127 or gamma + eps) would be far off
    assert np.abs(y - ref).max() < 1e-5 * np.abs(ref).max()


def test_bf16_output_is_rne_of_fp32(orc):
    import torch
    W, x = synth.tiny_inputs()
    gamma = orc.gamma(W)
    packed = orc.pack(orc.ternarize(W, gamma), 0)
    y32, _ = orc.forward(packed, 0, gamma, 512, 256, x, ydt=orc.F32)
    y16, _ = orc.forward(packed, 0, gamma, 512, 256, x, ydt=orc.BF16)
    ref = torch.from_numpy(y32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(y16, ref)


def test_bf16_conversion_specials(orc):
    import torch
    vals = np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.4e38, -1e-40, 1e-45,
                     np.inf, -np.inf], np.float32)
    rnd = synth.normal_f32(99, (4096,), 3.0)
    for v in np.concatenate([vals, rnd]):
        want = int(torch.tensor([v]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)[0])
        assert orc.f32_to_bf16(v) == want, v
        assert orc.bf16_to_f32(want) == np.float32(torch.tensor([v]).to(torch.bfloat16).float().item())


def test_pre_quantized_input(orc):
    """x given as int8 with its scales skips step 4 and reaches the same y."""
    W, x = synth.tiny_inputs()
    gamma = orc.gamma(W)
    packed = orc.pack(orc.ternarize(W, gamma), 0)
    xq, s = orc.act_quant(x)
    y1, _ = orc.forward(packed, 0, gamma, 512, 256, x)
    y2, _ = orc.forward(packed, 0, gamma, 512, 256, xq, scale=s)
    assert np.array_equal(y1, y2)


def test_zero_token_gives_zero(orc):
    W, _ = synth.tiny_inputs()
    gamma = orc.gamma(W)
    packed = orc.pack(orc.ternarize(W, gamma), 0)
    y, s = orc.forward(packed, 0, gamma, 512, 256, np.zeros((2, 256), np.float32))
    assert not y.any() and (s == np.float32(1e-6)).all()
