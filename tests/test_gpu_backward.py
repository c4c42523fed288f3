"""GPU parity of the STE backward through the C ABI against the oracle.

dW: both sides add in fp64 in token order and round once to fp32, so dW is
compared bit for bit.  dx: the oracle's sum over the rows is exact (no order),
rounded once to fp64; the kernel may add in any order, so dx is compared
within one fp32 ulp plus the fp64 rounding bound of an N-term sum
(gamma N 2^-52 sum |dy|), see ``assert_dx_close``."""
import numpy as np
import pytest
import torch

from bitlinear_b1_fwd_b200 import binding as B
from bitlinear_b1_fwd_b200 import synth
from gpu_helpers import dev, host, quantize_weights

pytestmark = pytest.mark.gpu

I2, T5, B1 = B.BL_PACK_I2, B.BL_PACK_T5, B.BL_PACK_B1


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bitlinear_b1_fwd_b200 import build
    build.build()
    assert torch.cuda.is_available()
    torch.cuda.init()


def _weights(orc, N, K, fmt, seed):
    W = synth.normal_f32(seed, (N, K), 0.02)
    if fmt == B1:
        Wd = dev(W)
        packed = torch.empty((N, B.bitlinear_packed_row_bytes(K, B1)), dtype=torch.uint8, device="cuda")
        beta = torch.empty(1, dtype=torch.float32, device="cuda")
        alpha = torch.empty(1, dtype=torch.float32, device="cuda")
        ws = torch.zeros(B.bitlinear_binarize_weights_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
        B.bitlinear_binarize_weights(Wd, packed, None, beta, alpha, ws)
        torch.cuda.synchronize()
        g, packed = np.float32(beta.item()), host(packed)
    else:
        g, _, packed = quantize_weights(W, fmt, codes=False)
    return g, packed, orc.unpack(packed, N, K, fmt)


def _widen(dy):
    return (dy.astype(np.uint32) << 16).view(np.float32) if dy.dtype == np.uint16 else dy


def assert_dx_close(dx, ref, codes, dy, g):
    """dx against the exact-sum oracle: a sum of N terms in fp64 in any order
    is within (N - 1) 2^-53 sum |term| of the exact sum; scaled by gamma (one
    more fp64 rounding) and rounded to fp32, two such values differ by at most
    one fp32 ulp of the larger plus gamma N 2^-52 sum |q dy|."""
    N = codes.shape[0]
    mag = np.abs(_widen(dy)).astype(np.float64) @ np.abs(codes).astype(np.float64)
    big = np.maximum(np.abs(dx), np.abs(ref)).astype(np.float32)
    tol = np.spacing(big).astype(np.float64) + float(g) * N * 2.0 ** -52 * mag
    err = np.abs(dx.astype(np.float64) - ref.astype(np.float64))
    bad = ~(err <= tol)
    assert not bad.any(), f"{bad.sum()} dx entries outside the bound; first at {np.argwhere(bad)[:3].tolist()}"
    # the bound is loose only where the sum cancels; report how many are bit-equal
    return float(np.mean(dx.view(np.uint32) == ref.view(np.uint32)))


def run_dx(packed, fmt, g, N, K, dy):
    M = dy.shape[0]
    dx = torch.full((M, K), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.bitlinear_backward_dx_workspace_bytes(M, N, K, fmt), dtype=torch.uint8, device="cuda")
    B.bitlinear_backward_dx(dev(packed), fmt, torch.tensor([float(g)], device="cuda"), N, K, dev(dy), dx, ws)
    torch.cuda.synchronize()
    assert B.bitlinear_device_status(ws) == B.BL_OK
    return host(dx)


@pytest.mark.parametrize("M,N,K,fmt,dydt", [
    (1, 512, 256, I2, "f32"),
    (3, 777, 1000, I2, "bf16"),     # K % 16 != 0: a partial last word; row blocks, the last partial
    (2, 3200, 3200, T5, "f32"),     # base 3 through the 2-bit transcoding
    (5, 300, 129, B1, "f32"),       # 1-bit (codes in {-1, +1}); three passes of two tokens
    (1, 8640, 3200, I2, "bf16"),    # 3B up-projection shape, one token
    (4, 1, 64, I2, "f32"),          # one row
    (128, 640, 512, I2, "bf16"),    # many tokens: 64 passes of two
    (1, 3200, 8640, I2, "f32"),     # 3B down-projection shape: 17 column blocks
    (2, 6001, 8192, I2, "bf16"),    # row blocks of 320 rows: three chunks of row pairs, odd last row
])
def test_backward_dx(orc, M, N, K, fmt, dydt):
    g, packed, codes = _weights(orc, N, K, fmt, 720 + K)
    dy = synth.normal_f32(721 + M, (M, N), 1e-3)
    if dydt == "bf16":
        dy = synth.to_bf16_bits(dy)
    dx = run_dx(packed, fmt, g, N, K, dy)
    ref = orc.backward_dx(codes, dy, g, parallel=True)
    assert_dx_close(dx, ref, codes, dy, g)


def run_dw(dy, xq, s, g, N, K):
    M = dy.shape[0]
    dw = torch.full((N, K), float("nan"), dtype=torch.float32, device="cuda")
    B.bitlinear_backward_dw(dev(dy), dev(xq), dev(s), torch.tensor([float(g)], device="cuda"), dw)
    torch.cuda.synchronize()
    return host(dw)


@pytest.mark.parametrize("M,N,K,dydt", [
    (1, 512, 256, "f32"),
    (3, 777, 1001, "bf16"),   # K % 4 != 0: scalar loads and stores
    (300, 64, 128, "f32"),    # two blocks of token factors
    (1, 3200, 3200, "bf16"),  # 3B attention shape, one token
    (1, 777, 1001, "f32"),    # one token (the per-row table kernel), K % 4 != 0
    (1, 5000, 64, "bf16"),    # one token, more rows than CTAs: each CTA refills its table per row
])
def test_backward_dw(orc, M, N, K, dydt):
    x = synth.entry_outliers(synth.normal_f32(730 + M, (M, K)), 731, 0.01, 20.0)
    xq, s = orc.act_quant(x)
    dy = synth.normal_f32(732 + M, (M, N), 1e-3)
    if dydt == "bf16":
        dy = synth.to_bf16_bits(dy)
    g = np.float32(0.0173)
    dw = run_dw(dy, xq, s, g, N, K)
    ref = orc.backward_dw(dy, xq, s, g)
    assert np.array_equal(dw.view(np.uint32), ref.view(np.uint32))


def test_backward_dw_one_token_every_code(orc):
    """One token whose codes take all 256 int8 values (including -128, which
    the API accepts though the quantizer never writes it), zero and negative
    gradients: every entry of the per-row table is used."""
    N, K = 300, 512
    xq = (np.arange(K) % 256 - 128).astype(np.int8).reshape(1, K)
    s = np.array([0.731], dtype=np.float32)
    dy = synth.normal_f32(740, (1, N), 1e-2)
    dy[0, ::7] = 0.0
    dy[0, 3] = -0.0
    g = np.float32(0.0419)
    dw = run_dw(dy, xq, s, g, N, K)
    ref = orc.backward_dw(dy, xq, s, g)
    assert np.array_equal(dw.view(np.uint32), ref.view(np.uint32))


def test_backward_dw_no_tokens_writes_zeros():
    N, K = 10, 16
    dw = torch.full((N, K), float("nan"), dtype=torch.float32, device="cuda")
    dy = torch.empty((0, N), dtype=torch.float32, device="cuda")
    xq = torch.empty((0, K), dtype=torch.int8, device="cuda")
    s = torch.empty((0,), dtype=torch.float32, device="cuda")
    B.bitlinear_backward_dw(dy, xq, s, torch.tensor([0.5], device="cuda"), dw)
    torch.cuda.synchronize()
    assert not host(dw).any()


def test_backward_after_forward_chain(orc):
    """The forward's own codes and scales feed dW: quantize, forward (bf16
    tokens), then both gradients, all through the C ABI."""
    M, N, K = 2, 640, 512
    W = synth.normal_f32(740, (N, K), 0.02)
    x = synth.to_bf16_bits(synth.normal_f32(741, (M, K)))
    g, _, packed = quantize_weights(W, I2, codes=False)
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    s = torch.empty((M,), dtype=torch.float32, device="cuda")
    B.bitlinear_quantize_acts(dev(x), xq, s)
    dy = synth.normal_f32(742, (M, N), 1e-2)
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    B.bitlinear_backward_dw(dev(dy), xq, s, torch.tensor([float(g)], device="cuda"), dw)
    dx = run_dx(packed, I2, g, N, K, dy)
    xq_ref, s_ref = orc.act_quant(x)
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(dw).view(np.uint32), orc.backward_dw(dy, xq_ref, s_ref, g).view(np.uint32))
    codes = orc.unpack(packed, N, K, I2)
    assert_dx_close(dx, orc.backward_dx(codes, dy, g), codes, dy, g)
