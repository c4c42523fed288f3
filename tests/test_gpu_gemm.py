"""GPU parity of the tensor-core path (more than four tokens, K a multiple of
16): every token-tile size, ragged N and K tails, base-3 weights (transcoded
to 2-bit), pre-quantized activations, the full 3B prefill, and the
bounded-wait error path."""
import numpy as np
import pytest
import torch

from bitlinear_b1_fwd_b200 import binding as B
from bitlinear_b1_fwd_b200 import synth
from gpu_helpers import assert_bf16_ulp, assert_f32_rel, dev, forward, host, quantize_weights

pytestmark = pytest.mark.gpu

I2, T5 = B.BL_PACK_I2, B.BL_PACK_T5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bitlinear_b1_fwd_b200 import build
    build.build()
    assert torch.cuda.is_available()


def ref_forward(orc, packed, fmt, g, N, K, x, ydt, scale=None, threads=True):
    """Oracle forward; the INT32 product runs on row slices in parallel."""
    if not threads:
        return orc.forward(packed, fmt, g, N, K, x, ydt=ydt, scale=scale)
    codes = orc.unpack(packed, N, K, fmt)
    if x.dtype == np.int8:
        xq, s = x, scale
    else:
        xq, s = orc.act_quant(x)
    acc = orc.matmul_i32(codes, xq, parallel=True)
    return orc.dequant(acc, g, s, ydt), s


def check(orc, packed, fmt, g, N, K, x, ydts=(B.BL_I32, B.BL_F32, B.BL_BF16), scale=None):
    for ydt in ydts:
        y, s = forward(packed, fmt, g, N, K, x, ydt, scale)
        y_ref, s_ref = ref_forward(orc, packed, fmt, g, N, K, x, ydt, scale)
        assert np.array_equal(s, s_ref)
        if ydt == B.BL_I32:
            bad = np.argwhere(y != y_ref)
            assert bad.size == 0, f"{len(bad)} INT32 mismatches, first {bad[:4].tolist()}"
        elif ydt == B.BL_F32:
            assert_f32_rel(y, y_ref)
        else:
            assert_bf16_ulp(y, y_ref)


@pytest.mark.parametrize("M", [5, 16, 17, 31, 32, 33, 64, 65, 127, 128, 129, 255, 256, 257, 600])
def test_token_tiles(orc, M):
    N, K = 300, 1024
    W = synth.normal_f32(81, (N, K), 0.02)
    x = synth.to_bf16_bits(synth.normal_f32(82 + M, (M, K)))
    g, _, packed = quantize_weights(W, I2, codes=False)
    check(orc, packed, I2, g, N, K, x)


@pytest.mark.parametrize("N,K,M", [(128, 16, 9), (129, 112, 20), (1, 144, 7), (257, 8640, 40),
                                   (640, 3200, 300), (100, 28672, 70), (8640, 128, 5)])
def test_ragged_shapes(orc, N, K, M):
    W = synth.normal_f32(N + 13 * K, (N, K), 0.02)
    x = synth.normal_f32(K + 7 * M, (M, K))
    g, _, packed = quantize_weights(W, I2, codes=False)
    check(orc, packed, I2, g, N, K, x)


@pytest.mark.parametrize("N,K,M", [(300, 1024, 40), (257, 8640, 9), (64, 8192, 300)])
def test_base3_through_transcode(orc, N, K, M):
    W = synth.normal_f32(N + 3 * K + 1, (N, K), 0.02)
    x = synth.to_bf16_bits(synth.normal_f32(K + M + 5, (M, K)))
    g, _, packed = quantize_weights(W, T5, codes=False)
    check(orc, packed, T5, g, N, K, x)


def test_prequantized_int8_input(orc):
    N, K, M = 384, 2048, 77
    W = synth.normal_f32(91, (N, K), 0.02)
    x = synth.normal_f32(92, (M, K))
    g, _, packed = quantize_weights(W, I2, codes=False)
    xq, s = orc.act_quant(x)
    check(orc, packed, I2, g, N, K, xq, scale=s)


def test_zero_tokens_and_zero_weights(orc):
    N, K, M = 256, 512, 48
    x = synth.normal_f32(93, (M, K))
    x[5] = 0.0
    x[47] = 0.0
    W = synth.normal_f32(94, (N, K), 0.02)
    g, _, packed = quantize_weights(W, I2, codes=False)
    check(orc, packed, I2, g, N, K, x)
    gz, _, pz = quantize_weights(np.zeros((N, K), np.float32), I2, codes=False)
    y, _ = forward(pz, I2, gz, N, K, x, B.BL_F32)
    assert not y.any()


def test_prefill_3b_full(orc):
    """3B prefill: 4096 tokens (bf16, 16 outlier channels x30) through the
    K=3200 -> N=8640 layer; every INT32 accumulator and bf16 output checked."""
    W, x = synth.prefill_3b_inputs()
    g, _, packed = quantize_weights(W, I2, codes=False)
    check(orc, packed, I2, g, 8640, 3200, x, ydts=(B.BL_I32, B.BL_BF16))


def test_block_3b_m128_m1024_sampled(orc):
    """The six 3B block layers at M = 128 (all tokens checked) and M = 1024
    (a seeded sample of 64 tokens checked against the oracle, since tokens are
    independent)."""
    rng = np.random.default_rng(7)
    for layer in range(6):
        c = synth.BLOCK_3B[layer]
        for M in (128, 1024):
            W, x = synth.block_3b_inputs(layer, M)
            g, _, packed = quantize_weights(W, I2, codes=False)
            y, s = forward(packed, I2, g, c["N"], c["K"], x, B.BL_I32)
            rows = np.arange(M) if M <= 128 else np.sort(rng.choice(M, 64, replace=False))
            y_ref, s_ref = ref_forward(orc, packed, I2, g, c["N"], c["K"], np.ascontiguousarray(x[rows]), B.BL_I32)
            assert np.array_equal(y[rows], y_ref)
            assert np.array_equal(s[rows], s_ref)


def test_wait_timeout_is_reported():
    """The tensor-core kernel with its producer switched off: every bounded
    wait runs out after about a millisecond, the kernel records the timeout
    and returns, and the context stays usable."""
    ws = torch.zeros(256 + 8192, dtype=torch.uint8, device="cuda")
    B.bitlinear_selftest_wait_timeout(ws)
    assert B.bitlinear_device_status(ws) == B.BL_ERR_DEVICE_TIMEOUT
    assert B.bitlinear_device_status(ws) == B.BL_OK
    # the device still works afterwards
    a = torch.ones(1024, device="cuda")
    assert float(a.sum().item()) == 1024.0
