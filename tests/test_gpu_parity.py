"""GPU parity: the CUDA path through the C ABI against the oracle, element by
element, on the seeded workloads and edge shapes.

Integers (gamma's bits, codes, packed bytes, x_q, scales, INT32 accumulators)
must be bit-exact; fp32 outputs within 1e-6 relative; bf16 outputs within 1 ulp.
"""
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
    torch.cuda.init()


def check_weights(orc, W, fmt):
    g, codes, packed = quantize_weights(W, fmt)
    g_ref = orc.gamma(W)
    assert g.view(np.uint32) == g_ref.view(np.uint32), (g, g_ref)
    codes_ref = orc.ternarize(W, g_ref, 1e-5, parallel=True)
    assert np.array_equal(codes, codes_ref)
    assert np.array_equal(packed, orc.pack(codes_ref, fmt))
    return g, packed


def check_forward(orc, packed, fmt, g, N, K, x, scale=None, ydts=(B.BL_I32, B.BL_F32, B.BL_BF16)):
    for ydt in ydts:
        y, s = forward(packed, fmt, g, N, K, x, ydt, scale)
        y_ref, s_ref = orc.forward(packed, fmt, g, N, K, x, ydt=ydt, scale=scale)
        assert np.array_equal(s, s_ref)
        if ydt == B.BL_I32:
            assert np.array_equal(y, y_ref)
        elif ydt == B.BL_F32:
            assert_f32_rel(y, y_ref)
        else:
            assert_bf16_ulp(y, y_ref)


# --- step 4: activation quantization ----------------------------------------------

def _act_cases():
    yield "tiny_f32_outliers", synth.tiny_inputs()[1]
    yield "3b_decode_bf16", synth.decode_3b_inputs(0)[1]
    yield "ragged_3x5_f32", synth.normal_f32(41, (3, 5))
    yield "ragged_17x129_bf16", synth.to_bf16_bits(synth.normal_f32(42, (17, 129)))
    yield "ragged_2x1000_f32", synth.normal_f32(43, (2, 1000))
    yield "ragged_5x7_bf16", synth.to_bf16_bits(synth.normal_f32(44, (5, 7)))
    z = synth.normal_f32(45, (4, 64))
    z[1] = 0.0
    z[2] = 1e-9
    yield "zero_and_tiny_rows", z
    # long rows: one 512-thread CTA per token (bf16 up to 32768, fp32 up to 16384
    # elements), and past that the warp-per-token kernel
    yield "70b_down_16x28672_bf16", synth.to_bf16_bits(
        synth.entry_outliers(synth.normal_f32(46, (16, 28672)), 47, 0.001, 30.0))
    yield "long_3x16384_f32", synth.normal_f32(48, (3, 16384))
    yield "long_2x32768_bf16", synth.to_bf16_bits(synth.normal_f32(49, (2, 32768)))
    yield "longer_2x40000_bf16", synth.to_bf16_bits(synth.normal_f32(50, (2, 40000)))
    yield "long_5x9000_f32", synth.normal_f32(51, (5, 9000))


@pytest.mark.parametrize("name,x", list(_act_cases()), ids=lambda v: v if isinstance(v, str) else "")
def test_quantize_acts(orc, name, x):
    M, K = x.shape
    xd = dev(x)
    xq = torch.full((M, K), 99, dtype=torch.int8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    B.bitlinear_quantize_acts(xd, xq, s)
    torch.cuda.synchronize()
    xq_ref, s_ref = orc.act_quant(x)
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(s), s_ref)


def test_quantize_acts_prefill_full(orc):
    """3B prefill activations: 4096 tokens x 3200 with 16 outlier channels."""
    _, x = synth.prefill_3b_inputs()
    xd = dev(x)
    xq = torch.empty((4096, 3200), dtype=torch.int8, device="cuda")
    s = torch.empty(4096, dtype=torch.float32, device="cuda")
    B.bitlinear_quantize_acts(xd, xq, s)
    torch.cuda.synchronize()
    xq_ref, s_ref = orc.act_quant(x)
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(s), s_ref)


def test_quantize_acts_round_half_even(orc):
    """Entries that land exactly on k + 0.5 after the multiply by 127."""
    xs = [np.float32(1.0)]
    for t in (0.5, 1.5, 2.5, 3.5, 126.5):
        v = np.float32(t / 127.0)
        for _ in range(400):
            r = np.float32(v * np.float32(127.0))
            if r == np.float32(t):
                break
            v = np.nextafter(v, np.float32(1) if r < t else np.float32(0))
        xs += [v, -v]
    x = np.array([xs + [0.0] * (16 - len(xs))], np.float32)
    xd = dev(x)
    xq = torch.empty_like(xd, dtype=torch.int8)
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    B.bitlinear_quantize_acts(xd, xq, s)
    torch.cuda.synchronize()
    assert host(xq)[0, :11].tolist() == [127, 0, 0, 2, -2, 2, -2, 4, -4, 126, -126]
    assert np.array_equal(host(xq), orc.act_quant(x)[0])


# --- steps 1-3: weights -------------------------------------------------------------

def test_worked_examples(orc):
    for W, codes in ((synth.EXAMPLE_A, [0, -1, 1, -1, 0]), (synth.EXAMPLE_B, [1, -1, 0, -1, 1])):
        for fmt in (I2, T5):
            g, c, p = quantize_weights(W, fmt)
            assert c[0].tolist() == codes
            assert g == orc.gamma(W)
            assert np.array_equal(p, orc.pack(c, fmt))


def _weight_cases():
    yield "tiny", synth.tiny_inputs()[0]
    yield "ragged_3x7", synth.normal_f32(51, (3, 7), 0.02)
    yield "ragged_5x129", synth.normal_f32(52, (5, 129), 0.02)
    yield "ragged_2x8193", synth.normal_f32(53, (2, 8193), 0.02)
    yield "one", np.array([[0.3]], np.float32)
    yield "ragged_7x81", synth.normal_f32(54, (7, 81), 1.0)
    yield "bf16_300x1000", synth.to_bf16_bits(synth.normal_f32(55, (300, 1000), 0.02))
    yield "bf16_ragged_9x77", synth.to_bf16_bits(synth.normal_f32(56, (9, 77), 0.02))
    yield "zeros", np.zeros((4, 100), np.float32)
    yield "many_chunks_40x100003", synth.normal_f32(57, (40, 100003), 0.01)


@pytest.mark.parametrize("fmt", [I2, T5])
@pytest.mark.parametrize("name,W", list(_weight_cases()), ids=lambda v: v if isinstance(v, str) else "")
def test_quantize_weights(orc, name, W, fmt):
    check_weights(orc, W, fmt)


@pytest.mark.parametrize("layer", [0, 1])
def test_quantize_weights_3b(orc, layer):
    W, _ = synth.decode_3b_inputs(layer)
    check_weights(orc, W, I2)
    if layer == 0:
        check_weights(orc, W, T5)


def test_ternarize_threshold_boundary(orc):
    """A fixed gamma and weights planted at and next to d/2 = (gamma + eps)/2:
    the codes must equal the oracle's IEEE-division codes at the boundary."""
    gamma = np.float32(0.0163)
    d = np.float32(gamma + np.float32(1e-5))
    half = np.float32(d / np.float32(2))
    plant = [half, -half, np.float32(0), np.float32(-0.0), d, -d, np.float32(1.5) * d]
    v = half
    for _ in range(64):  # the fp32 values just above d/2
        v = np.nextafter(v, np.float32(1))
        plant += [v, -v]
    v = half
    for _ in range(16):
        v = np.nextafter(v, np.float32(0))
        plant += [v, -v]
    W = synth.normal_f32(61, (3, 1000), 0.02)
    W[0, :len(plant)] = plant
    # exactly d/2 divides to 0.5 (-> 0); every fp32 above it divides to more than 0.5
    assert np.float32(half / d) == np.float32(0.5)
    assert all(np.float32(abs(p) / d) > np.float32(0.5) for p in plant[7:7 + 128])
    for fmt in (I2, T5):
        Wd = dev(W)
        g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
        packed = torch.empty((3, B.bitlinear_packed_row_bytes(1000, fmt)), dtype=torch.uint8, device="cuda")
        codes = torch.empty((3, 1000), dtype=torch.int8, device="cuda")
        B.bitlinear_ternarize_pack(Wd, g, 1e-5, fmt, packed, codes)
        torch.cuda.synchronize()
        ref = orc.ternarize(W, gamma, 1e-5)
        assert np.array_equal(host(codes), ref)
        assert np.array_equal(host(packed), orc.pack(ref, fmt))


def test_pack_and_bad_codes(orc):
    rng = np.random.default_rng(3)
    for (N, K) in [(5, 3), (7, 129), (64, 3200), (3, 8193), (3, 48), (9, 4096)]:
        codes = rng.integers(-1, 2, (N, K), dtype=np.int8)
        for fmt in (I2, T5):
            packed = torch.empty((N, B.bitlinear_packed_row_bytes(K, fmt)), dtype=torch.uint8, device="cuda")
            ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
            B.bitlinear_pack(dev(codes), fmt, packed, ws)
            assert B.bitlinear_device_status(ws) == B.BL_OK
            assert np.array_equal(host(packed), orc.pack(codes, fmt))
    bad = rng.integers(-1, 2, (4, 40), dtype=np.int8)
    bad[2, 17] = 3
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    packed = torch.empty((4, 16), dtype=torch.uint8, device="cuda")
    B.bitlinear_pack(dev(bad), I2, packed, ws)
    assert B.bitlinear_device_status(ws) == B.BL_ERR_BAD_CODE
    assert B.bitlinear_device_status(ws) == B.BL_OK      # read clears the flag
    fixed = bad.copy()
    fixed[2, 17] = 0
    assert np.array_equal(host(packed), orc.pack(fixed, I2))
    # the same with K % 16 == 0 (codes read 16 at a time), both formats
    for fmt in (I2, T5):
        bad = rng.integers(-1, 2, (3, 80), dtype=np.int8)
        bad[1, 66] = -2
        ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        packed = torch.empty((3, B.bitlinear_packed_row_bytes(80, fmt)), dtype=torch.uint8, device="cuda")
        B.bitlinear_pack(dev(bad), fmt, packed, ws)
        assert B.bitlinear_device_status(ws) == B.BL_ERR_BAD_CODE
        fixed = bad.copy()
        fixed[1, 66] = 0
        assert np.array_equal(host(packed), orc.pack(fixed, fmt))


# --- steps 4-6: forward ------------------------------------------------------------

@pytest.mark.parametrize("fmt", [I2, T5])
def test_forward_tiny(orc, fmt):
    W, x = synth.tiny_inputs()
    g, packed = check_weights(orc, W, fmt)
    check_forward(orc, packed, fmt, g, 512, 256, x)


def test_forward_worked_example(orc):
    g, _, packed = quantize_weights(synth.EXAMPLE_A, I2)
    y, s = forward(packed, I2, g, 1, 5, np.ones((1, 5), np.float32), B.BL_I32)
    assert y.tolist() == [[-127]] and s.tolist() == [1.0]
    y, _ = forward(packed, I2, g, 1, 5, np.ones((1, 5), np.float32), B.BL_F32)
    assert abs(float(y[0, 0]) + 0.61) < 1e-6


@pytest.mark.parametrize("layer", [0, 1])
@pytest.mark.parametrize("fmt", [I2, T5])
def test_forward_3b_decode(orc, layer, fmt):
    W, x = synth.decode_3b_inputs(layer)
    c = synth.DECODE_3B[layer]
    g, _, packed = quantize_weights(W, fmt, codes=False)
    check_forward(orc, packed, fmt, g, c["N"], c["K"], x)


@pytest.mark.parametrize("fmt", [I2, T5])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 16, 17])
def test_forward_token_counts(orc, fmt, M):
    W = synth.normal_f32(71, (300, 1000), 0.02)
    x = synth.to_bf16_bits(synth.normal_f32(72, (M, 1000)))
    g, _, packed = quantize_weights(W, fmt, codes=False)
    check_forward(orc, packed, fmt, g, 300, 1000, x)


@pytest.mark.parametrize("fmt", [I2, T5])
@pytest.mark.parametrize("N,K,M", [(1, 1, 1), (3, 5, 2), (33, 7, 3), (65, 129, 1), (17, 8193, 2),
                                   (129, 4097, 4), (2, 20001, 1)])
def test_forward_ragged(orc, fmt, N, K, M):
    W = synth.normal_f32(N * 7 + K, (N, K), 0.02)
    x = synth.normal_f32(K * 3 + M, (M, K))
    g, _, packed = quantize_weights(W, fmt, codes=False)
    check_forward(orc, packed, fmt, g, N, K, x)


def test_forward_prequantized_and_degenerate(orc):
    W, x = synth.tiny_inputs()
    g, _, packed = quantize_weights(W, I2, codes=False)
    xq, s = orc.act_quant(x)
    check_forward(orc, packed, I2, g, 512, 256, xq, scale=s)
    # zero tokens, and an all-zero weight matrix (gamma 0)
    xz = x.copy()
    xz[3] = 0.0
    check_forward(orc, packed, I2, g, 512, 256, xz)
    gz, _, pz = quantize_weights(np.zeros((64, 256), np.float32), T5, codes=False)
    assert gz == 0.0
    y, _ = forward(pz, T5, gz, 64, 256, x, B.BL_F32)
    assert not y.any()
    # M = 0 launches nothing and returns success
    y, _ = forward(packed, I2, g, 512, 256, np.zeros((0, 256), np.float32), B.BL_F32)
    assert y.shape == (0, 512)


@pytest.mark.parametrize("M", [1, 16])
def test_forward_3b_block(orc, M):
    """The six BitLinears of a 3B block (Q, K, V, O, up, down), each with its
    own per-token quantization, at M = 1 and 16 tokens."""
    for layer in range(6):
        W, x = synth.block_3b_inputs(layer, M)
        c = synth.BLOCK_3B[layer]
        g, _, packed = quantize_weights(W, I2, codes=False)
        check_forward(orc, packed, I2, g, c["N"], c["K"], x, ydts=(B.BL_I32, B.BL_BF16))


def test_misaligned_pointer_rejected():
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    xq = torch.zeros(64, dtype=torch.int8, device="cuda")
    s = torch.zeros(2, dtype=torch.float32, device="cuda")
    with pytest.raises(B.BitLinearError) as e:
        B.bitlinear_quantize_acts(x[1:33].view(1, 32), xq[:32].view(1, 32), s[:1])
    assert e.value.status == B.BL_ERR_MISALIGNED


def test_quantize_acts_near_ties(orc):
    """Entries whose quotient x / s * 127 lands within a few fp32 ulps of a
    half-integer, at several token scales: the cases the kernel settles with
    the exact quotient.  Both the standalone quantizer and the GEMV prologue."""
    rows = []
    for smax in (1.0, 3.7, 0.013, 250.0, 1e-6):
        xs = [np.float32(smax)]
        for t in (0.5, 1.5, 2.5, 63.5, 100.5, 126.5):
            v0 = np.float32(t / 127.0 * smax)
            up, dn = v0, v0
            xs += [v0, -v0]
            for _ in range(12):
                up = np.nextafter(up, np.float32(np.inf))
                dn = np.nextafter(dn, np.float32(0))
                xs += [up, -up, dn, -dn]
        rows.append(xs)
    width = max(len(r) for r in rows)
    width += (-width) % 16
    x = np.zeros((len(rows), width), np.float32)
    for i, r in enumerate(rows):
        x[i, :len(r)] = r
    xq_ref, s_ref = orc.act_quant(x)
    xd = dev(x)
    xq = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    s = torch.empty(x.shape[0], dtype=torch.float32, device="cuda")
    B.bitlinear_quantize_acts(xd, xq, s)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(s), s_ref)
    # the decode path quantizes in its prologue: an identity-like weight matrix
    # (row n has +1 at column n) makes y[:, n] = x_q[:, n] for n < K
    K = x.shape[1]
    codes = np.zeros((K, K), np.int8)
    np.fill_diagonal(codes, 1)
    packed = orc.pack(codes, I2)
    for m in range(x.shape[0]):
        y, sm = forward(packed, I2, np.float32(1.0), K, K, x[m:m + 1], B.BL_I32)
        assert np.array_equal(y[0], xq_ref[m].astype(np.int32))
        assert sm[0] == s_ref[m]


# --- one-token base-3 decode: the column-stationary kernel and its limits ---------

@pytest.mark.parametrize("N,K,xkind", [(300, 1000, "int8"), (65, 129, "int8"), (97, 8193, "bf16"),
                                       (37, 61440, "bf16"), (37, 61441, "f32"), (5, 80 * 33, "f32")])
def test_forward_t5_one_token(orc, N, K, xkind):
    """Rows of 1..768 segments (the kernel's limit: 61440 weights) and one past
    it (the general kernel), ragged K, fp32 / bf16 tokens quantized inside and
    int8 tokens with their given scale."""
    W = synth.normal_f32(N * 13 + K, (N, K), 0.02)
    x = synth.normal_f32(K * 5 + N, (1, K))
    g, _, packed = quantize_weights(W, T5, codes=False)
    if xkind == "int8":
        xq, s = orc.act_quant(x)
        check_forward(orc, packed, T5, g, N, K, xq, scale=s)
    else:
        check_forward(orc, packed, T5, g, N, K, synth.to_bf16_bits(x) if xkind == "bf16" else x)


def test_forward_t5_many_rows_per_cta(orc):
    """More rows than one CTA's row sums hold (N > 148 x 1024 on a B200): the
    general kernel takes the call, with the same results."""
    N, K = 160_000, 40
    W = synth.normal_f32(91, (N, K), 0.02)
    x = synth.normal_f32(92, (1, K))
    g, _, packed = quantize_weights(W, T5, codes=False)
    check_forward(orc, packed, T5, g, N, K, x, ydts=(B.BL_I32, B.BL_BF16))


# --- one-token 2-bit decode: the lean kernel and its limits ----------------------------

@pytest.mark.parametrize("N,K,xkind", [(300, 1000, "int8"), (150, 4104, "int8"), (97, 8193, "bf16"),
                                       (149, 32768, "bf16"), (37, 32769, "f32"), (5, 64, "f32"),
                                       (2000, 2048, "bf16")])
def test_forward_i2_one_token(orc, N, K, xkind):
    """Rows of 16 B .. 8 KB (the lean kernel's limit: K = 32768) and one past
    it (the general kernel), CTAs with one to many rows, ragged K, fp32 / bf16
    tokens quantized inside and int8 tokens with their given scale."""
    W = synth.normal_f32(N * 11 + K, (N, K), 0.02)
    x = synth.normal_f32(K * 7 + N, (1, K))
    g, _, packed = quantize_weights(W, I2, codes=False)
    if xkind == "int8":
        xq, s = orc.act_quant(x)
        check_forward(orc, packed, I2, g, N, K, xq, scale=s)
    else:
        check_forward(orc, packed, I2, g, N, K, synth.to_bf16_bits(x) if xkind == "bf16" else x)


def test_forward_i2_many_rows_per_cta(orc):
    """More rows than one CTA's row sums hold: the lean kernel's row tiles."""
    N, K = 160_000, 64
    W = synth.normal_f32(93, (N, K), 0.02)
    x = synth.to_bf16_bits(synth.normal_f32(94, (1, K)))
    g, _, packed = quantize_weights(W, I2, codes=False)
    check_forward(orc, packed, I2, g, N, K, x, ydts=(B.BL_I32, B.BL_BF16))


# --- pre-norm: LayerNorm of each token, then per-token INT8 ---------------------------

def _ln_cases():
    yield "tiny_f32_outliers", synth.tiny_inputs()[1]
    yield "3b_decode_bf16", synth.decode_3b_inputs(0)[1]
    yield "3b_prefill_bf16_outlier_channels", synth.prefill_3b_inputs()[1]
    yield "ragged_3x20001_f32", synth.normal_f32(71, (3, 20001))
    yield "k1_f32", synth.normal_f32(72, (4, 1))
    yield "70b_down_bf16", synth.to_bf16_bits(synth.normal_f32(73, (2, 28672)))
    # the register form's three widths (K <= 2048, <= 3328, <= 4096), fp32 input,
    # more tokens than resident CTAs (each CTA loads its next token ahead)
    yield "1300x2048_f32", synth.normal_f32(75, (1300, 2048))
    yield "900x3000_f32", synth.entry_outliers(synth.normal_f32(76, (900, 3000)), 77, 0.01, 20.0)
    yield "700x4096_bf16", synth.to_bf16_bits(synth.normal_f32(78, (700, 4096)))
    yield "5x3330_f32", synth.normal_f32(79, (5, 3330))
    c = synth.normal_f32(74, (4, 300))
    c[1] = 0.375  # a constant token: y = ln_b
    c[2] = 0.0
    yield "constant_and_zero_tokens", c


@pytest.mark.parametrize("name,x", list(_ln_cases()), ids=lambda v: v if isinstance(v, str) else "")
def test_layernorm_quantize_acts(orc, name, x):
    """bf16 LayerNorm output, INT8 codes and scales bit-exact against the oracle."""
    M, K = x.shape
    g = synth.normal_f32(80 + K % 11, (K,), 1.0)
    b = synth.normal_f32(81 + K % 13, (K,), 0.1)
    y_ref, xq_ref, s_ref = orc.layernorm_quant(x, g, b, 1e-5)
    y = torch.empty((M, K), dtype=torch.int16, device="cuda")
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    s = torch.empty((M,), dtype=torch.float32, device="cuda")
    B.bitlinear_layernorm_quantize_acts(dev(x), dev(g), dev(b), 1e-5, xq, s, y)
    torch.cuda.synchronize()
    assert np.array_equal(host(y).view(np.uint16), y_ref)
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(s).view(np.uint32), s_ref.view(np.uint32))


def test_layernorm_quantize_acts_feeds_forward(orc):
    """The codes and scales go straight into the forward as int8 tokens."""
    W, x = synth.decode_3b_inputs(0)
    c = synth.DECODE_3B[0]
    K = c["K"]
    g = synth.normal_f32(90, (K,), 1.0)
    b = synth.normal_f32(91, (K,), 0.1)
    _, xq_ref, s_ref = orc.layernorm_quant(x, g, b, 1e-5)
    xq = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    s = torch.empty((x.shape[0],), dtype=torch.float32, device="cuda")
    B.bitlinear_layernorm_quantize_acts(dev(x), dev(g), dev(b), 1e-5, xq, s)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref)
    gam, _, packed = quantize_weights(W, I2, codes=False)
    check_forward(orc, packed, I2, gam, c["N"], K, xq_ref, scale=s_ref)


# --- several layers sharing their input (a block's Q, K, V projections) -------------

def _grouped_weights(orc, rows, K, fmt, seed):
    """Each group quantized on its own (its own gamma); packed rows concatenated."""
    gammas, packs = [], []
    for i, n in enumerate(rows):
        W = synth.normal_f32(seed + i, (n, K), 0.02 * (i + 1))
        g, _, packed = quantize_weights(W, fmt, codes=False)
        gammas.append(g)
        packs.append(packed)
    return np.array(gammas, np.float32), np.concatenate(packs, axis=0)


def check_forward_grouped(orc, rows, K, fmt, x, scale=None, ydts=(B.BL_I32, B.BL_F32, B.BL_BF16)):
    gammas, packed = _grouped_weights(orc, rows, K, fmt, 300 + K)
    M, N = x.shape[0], sum(rows)
    for ydt in ydts:
        xd = dev(x)
        sd = dev(scale) if scale is not None else torch.full((M,), -1.0, dtype=torch.float32, device="cuda")
        tdt = {B.BL_F32: torch.float32, B.BL_BF16: torch.bfloat16, B.BL_I32: torch.int32}[ydt]
        y = torch.empty((M, N), dtype=tdt, device="cuda")
        y.view(torch.uint8).fill_(0xCD)
        need = B.bitlinear_forward_grouped_workspace_bytes(M, rows, K, fmt, B.dtype_code(xd))
        ws = torch.zeros(max(256, need), dtype=torch.uint8, device="cuda")
        B.bitlinear_forward_grouped(dev(packed), fmt, dev(gammas), rows, K, xd, sd, y, ws)
        torch.cuda.synchronize()
        assert B.bitlinear_device_status(ws) == B.BL_OK
        yh, sh = host(y), host(sd)
        off = 0
        for g, n in enumerate(rows):
            y_ref, s_ref = orc.forward(packed[off:off + n], fmt, gammas[g], n, K, x, ydt=ydt, scale=scale)
            assert np.array_equal(sh, s_ref)
            got = yh[:, off:off + n]
            if ydt == B.BL_I32:
                assert np.array_equal(got, y_ref), (g, n)
            elif ydt == B.BL_F32:
                assert_f32_rel(got, y_ref)
            else:
                assert_bf16_ulp(got, y_ref)
            off += n
        assert off == N


@pytest.mark.parametrize("M", [1, 3, 4, 5, 16, 40, 130])
@pytest.mark.parametrize("fmt", [I2, T5])
def test_forward_grouped_qkv(orc, M, fmt):
    """Three groups of ragged sizes (unaligned column offsets included), one
    GEMV launch for up to 4 tokens, one product per group beyond."""
    K = 640
    x = synth.to_bf16_bits(synth.normal_f32(310 + M, (M, K)))
    check_forward_grouped(orc, [200, 72, 131], K, fmt, x)


def test_forward_grouped_aligned_columns_int8_tokens(orc):
    """Row counts that keep every group's columns 16-byte aligned (the tensor
    map store path), int8 tokens with given scales."""
    M, K = 24, 1024
    xf = synth.normal_f32(320, (M, K))
    xq, s = orc.act_quant(xf)
    check_forward_grouped(orc, [256, 128, 384], K, I2, xq.astype(np.int8), scale=s)


def test_forward_grouped_one_group_matches_forward(orc):
    """A single group is the plain forward."""
    K, n = 512, 333
    x = synth.normal_f32(321, (2, K))
    check_forward_grouped(orc, [n], K, T5, x)


def test_forward_grouped_eight_groups_decode(orc):
    """The most groups one call takes, at one token, with one-row groups in it."""
    K = 384
    x = synth.to_bf16_bits(synth.normal_f32(322, (1, K)))
    check_forward_grouped(orc, [1, 64, 3, 128, 1, 200, 17, 90], K, I2, x)


def test_forward_grouped_rejects_bad_groups():
    g = torch.ones(9, dtype=torch.float32, device="cuda")
    x = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    y = torch.empty((1, 9), dtype=torch.float32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    p = torch.zeros((9, 16), dtype=torch.uint8, device="cuda")
    for rows in ([1] * 9, [3, 0, 6], []):
        with pytest.raises(B.BitLinearError) as e:
            B.bitlinear_forward_grouped(p, I2, g, rows, 64, x, s, y, ws)
        assert e.value.status == B.BL_ERR_INVALID_VALUE
