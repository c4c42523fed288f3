"""GPU parity of the one-token decode GEMVs (the column-stationary kernels
with K % 16 == 0: 2-bit rows of up to 8 KB, and base-3 and 1-bit rows where
the table, token, codes and ring fit) against the oracle.

The cases walk its geometry: segments per row from 1 to 512 (several rows per
warp, warps that span two rows, one row per warp), one to about a thousand
rows per CTA, one to four 16-element token chunks per thread, fp32 / bf16
tokens quantized inside and int8 tokens with their given scale, zero tokens,
and the row-group table of the grouped forward.  INT32 accumulators and the
scale bit for bit, fp32 y within 1e-6 relative, bf16 y within 1 ulp."""
import numpy as np
import pytest
import torch

from bitlinear_b1_fwd_b200 import binding as B
from bitlinear_b1_fwd_b200 import synth
from gpu_helpers import assert_bf16_ulp, assert_f32_rel, dev, forward, host, quantize_weights

pytestmark = pytest.mark.gpu

I2 = B.BL_PACK_I2
T5 = B.BL_PACK_T5
B1 = B.BL_PACK_B1


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bitlinear_b1_fwd_b200 import build
    build.build()
    assert torch.cuda.is_available()
    torch.cuda.init()


def _check(orc, N, K, xkind, seed, zero_token=False, ydts=(B.BL_I32, B.BL_F32, B.BL_BF16), fmt=I2):
    W = synth.normal_f32(seed, (N, K), 0.02)
    x = synth.entry_outliers(synth.normal_f32(seed + 1, (1, K)), seed + 2, 0.01, 20.0)
    if zero_token:
        x[:] = 0.0
    if fmt == B1:  # the 1-bit variant: beta in gamma's place
        N_, K_ = W.shape
        packed_t = torch.empty((N_, B.bitlinear_packed_row_bytes(K_, B1)), dtype=torch.uint8, device="cuda")
        beta = torch.empty((1,), dtype=torch.float32, device="cuda")
        alpha = torch.empty((1,), dtype=torch.float32, device="cuda")
        ws = torch.zeros(B.bitlinear_binarize_weights_workspace_bytes(N_, K_), dtype=torch.uint8, device="cuda")
        B.bitlinear_binarize_weights(dev(W), packed_t, None, beta, alpha, ws)
        torch.cuda.synchronize()
        g, packed = np.float32(beta.item()), host(packed_t)
    else:
        g, _, packed = quantize_weights(W, fmt, codes=False)
    scale = None
    if xkind == "int8":
        x, scale = orc.act_quant(x)
    elif xkind == "bf16":
        x = synth.to_bf16_bits(x)
    for ydt in ydts:
        y, s = forward(packed, fmt, g, N, K, x, ydt, scale)
        y_ref, s_ref = orc.forward(packed, fmt, g, N, K, x, ydt=ydt, scale=scale)
        assert np.array_equal(s, s_ref)
        if ydt == B.BL_I32:
            assert np.array_equal(y, y_ref), np.argwhere(y != y_ref)[:5].tolist()
        elif ydt == B.BL_F32:
            assert_f32_rel(y, y_ref)
        else:
            assert_bf16_ulp(y, y_ref)


@pytest.mark.parametrize("N,K", [
    (300, 64),      # one segment per row: 32 rows per warp
    (1000, 192),    # 3 segments per row, a warp spans 11 rows
    (777, 1088),    # 17 segments: warps span two or three rows
    (8640, 3200),   # 3B up: 50 segments, 10 rows per step
    (3200, 8640),   # 3B down: 135 segments, three rows per step, two chunks per thread
    (900, 8192),    # 128 segments: four rows per step, one row per warp
    (500, 16448),   # 257 segments: one row per step, four chunks per thread
    (160, 28672),   # 70B down rows: 448 segments
    (149, 32768),   # 512 segments (int8 tokens fit in shared memory)
])
@pytest.mark.parametrize("xkind", ["bf16", "f32", "int8"])
def test_gemv1_geometry(orc, N, K, xkind):
    _check(orc, N, K, xkind, seed=N * 13 + K)


@pytest.mark.parametrize("N", [1, 5, 147, 148, 149, 296, 150_000])
def test_gemv1_rows_per_cta(orc, N):
    """From one row on a few CTAs to about a thousand rows per CTA (row sums
    held in shared memory), at 3 and 50 segments per row."""
    for K in (192, 3200) if N < 100_000 else (192,):
        _check(orc, N, K, "bf16", seed=N + K, ydts=(B.BL_I32, B.BL_BF16))


def test_gemv1_zero_token(orc):
    _check(orc, 640, 3200, "bf16", seed=5, zero_token=True)
    _check(orc, 640, 3200, "f32", seed=6, zero_token=True)


def test_gemv1_3b_layers_back_to_back(orc):
    """The two 3B decode layers chained on one stream without host syncs (each
    launch may start while the previous one still runs): the second layer's
    input is the first layer's output."""
    (Wu, xu), (Wd, _) = synth.decode_3b_inputs(0), synth.decode_3b_inputs(1)
    gu, _, pu = quantize_weights(Wu, I2, codes=False)
    gd, _, pd = quantize_weights(Wd, I2, codes=False)
    Nu, Ku = Wu.shape
    Nd, Kd = Wd.shape
    assert Ku == Nd and Kd == Nu
    x0 = dev(xu)
    h = torch.empty((1, Nu), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((1, Nd), dtype=torch.bfloat16, device="cuda")
    s1 = torch.empty(1, dtype=torch.float32, device="cuda")
    s2 = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    gud = torch.tensor([float(gu)], device="cuda")
    gdd = torch.tensor([float(gd)], device="cuda")
    pud, pdd = dev(pu), dev(pd)
    for _ in range(3):
        B.bitlinear_forward(pud, I2, gud, Nu, Ku, x0, s1, h, ws)
        B.bitlinear_forward(pdd, I2, gdd, Nd, Kd, h, s2, out, ws)
    torch.cuda.synchronize()
    assert B.bitlinear_device_status(ws) == B.BL_OK
    h_ref, _ = orc.forward(pu, I2, gu, Nu, Ku, xu, ydt=B.BL_BF16)
    assert_bf16_ulp(host(h), h_ref)
    # the second layer against the oracle on the GPU's own h (1 ulp of h may
    # move a code, so the reference takes the same bf16 input)
    out_ref, _ = orc.forward(pd, I2, gd, Nd, Kd, host(h), ydt=B.BL_BF16)
    assert_bf16_ulp(host(out), out_ref)


@pytest.mark.parametrize("N,K", [
    (300, 64),      # one base-3 segment per row (80 weights, 16 of them padding)
    (1000, 400),    # 5 segments: a warp spans several rows
    (777, 1600),    # 20 segments
    (8640, 3200),   # 3B up: 40 segments, 8 rows per step
    (3200, 8640),   # 3B down: 108 segments, two chunks per thread
    (900, 8192),    # 70B up rows: 103 segments, four rows per step, 6 ring stages
    (500, 12800),   # 160 segments: three rows of 160 lanes per step
    (149, 20480),   # 256 segments (int8 tokens only: bf16 and fp32 ones take the other kernel)
])
@pytest.mark.parametrize("xkind", ["bf16", "f32", "int8"])
def test_gemv1_t5_geometry(orc, N, K, xkind):
    """Base-3 rows in the column-stationary layout (and, where the token does
    not fit beside the table, the fallback kernel)."""
    _check(orc, N, K, xkind, seed=N * 17 + K, fmt=T5)


def test_gemv1_t5_zero_token_and_rows_per_cta(orc):
    _check(orc, 640, 3200, "bf16", seed=7, zero_token=True, fmt=T5)
    for N in (1, 149, 30_000):
        _check(orc, N, 400, "bf16", seed=N, fmt=T5, ydts=(B.BL_I32, B.BL_BF16))


@pytest.mark.parametrize("N,K", [
    (300, 128),     # one 1-bit segment per row (128 weights)
    (1000, 1024),   # 8 segments
    (777, 3200),    # 25 segments: a warp spans two rows
    (900, 8192),    # 70B up rows: 64 segments, 8 rows per step
    (3200, 8640),   # 68 segments in 96 lanes per row, two chunks per thread
    (500, 16384),   # 128 segments, two chunks per thread
    (160, 28672),   # 70B down rows: four chunks per thread, so the lean kernel
])
@pytest.mark.parametrize("xkind", ["bf16", "f32", "int8"])
def test_gemv1_b1_geometry(orc, N, K, xkind):
    """1-bit rows in the column-stationary layout (bit-plane codes in
    registers), and past its limit the lean kernel."""
    _check(orc, N, K, xkind, seed=N * 19 + K, fmt=B1)


def test_gemv1_b1_zero_token_and_rows_per_cta(orc):
    _check(orc, 640, 3200, "bf16", seed=9, zero_token=True, fmt=B1)
    for N in (1, 149, 30_000):
        _check(orc, N, 1024, "bf16", seed=N + 3, fmt=B1, ydts=(B.BL_I32, B.BL_BF16))
