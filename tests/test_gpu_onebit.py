"""GPU parity of the 1-bit variant through the C ABI against the oracle:
alpha, beta, the {-1, +1} codes and their 8-per-byte packing bit-exact; the
forward (1-bit GEMV for up to 4 tokens, the tensor-core path beyond, rows too
long for the 1-bit GEMV through the 2-bit transcoding) integers exact, fp32
within 1e-6 relative, bf16 within 1 ulp."""
import numpy as np
import pytest
import torch

from bitlinear_b1_fwd_b200 import binding as B
from bitlinear_b1_fwd_b200 import synth
from gpu_helpers import assert_bf16_ulp, assert_f32_rel, dev, forward, host

pytestmark = pytest.mark.gpu

B1 = B.BL_PACK_B1


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bitlinear_b1_fwd_b200 import build
    build.build()
    assert torch.cuda.is_available()
    torch.cuda.init()


def binarize(W: np.ndarray, codes: bool = True):
    Wd = dev(W)
    N, K = W.shape
    packed = torch.full((N, B.bitlinear_packed_row_bytes(K, B1)), 0xAB, dtype=torch.uint8, device="cuda")
    cd = torch.full((N, K), 77, dtype=torch.int8, device="cuda") if codes else None
    beta = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    alpha = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.bitlinear_binarize_weights_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
    B.bitlinear_binarize_weights(Wd, packed, cd, beta, alpha, ws)
    torch.cuda.synchronize()
    assert B.bitlinear_device_status(ws) == B.BL_OK
    return (np.float32(alpha.item()), np.float32(beta.item()), host(cd) if codes else None, host(packed))


def _weight_cases():
    yield "example_b_1x5_f32", synth.EXAMPLE_B
    yield "tiny_512x256_f32", synth.tiny_inputs()[0]
    yield "3b_3200x3200_bf16", synth.to_bf16_bits(synth.normal_f32(600, (3200, 3200), 0.02))
    yield "ragged_37x3001_f32", synth.normal_f32(601, (37, 3001), 0.02) + np.float32(0.003)
    yield "ragged_5x129_bf16", synth.to_bf16_bits(synth.normal_f32(602, (5, 129), 1.0))
    yield "k1_9x1_f32", synth.normal_f32(603, (9, 1), 1.0)
    t = np.zeros((4, 64), np.float32)
    t[1, :] = 2.0  # alpha = 0.5: the zeros go to -1, the twos to +1
    yield "two_levels_4x64_f32", t


@pytest.mark.parametrize("name,W", list(_weight_cases()), ids=lambda v: v if isinstance(v, str) else "")
def test_binarize_weights(orc, name, W):
    a, b, codes, packed = binarize(W)
    a_ref, b_ref, codes_ref = orc.binarize_weights(W)
    assert a.view(np.uint32) == a_ref.view(np.uint32), (a, a_ref)
    assert b.view(np.uint32) == b_ref.view(np.uint32), (b, b_ref)
    assert np.array_equal(codes, codes_ref)
    assert np.array_equal(packed, orc.pack(codes_ref, B1))


def test_binarize_packed_only_matches(orc):
    W = synth.normal_f32(604, (300, 1000), 0.02)
    a, b, _, packed = binarize(W, codes=False)
    _, _, codes_ref = orc.binarize_weights(W)
    assert np.array_equal(packed, orc.pack(codes_ref, B1))


def test_pack_b1_from_codes(orc):
    rng = np.random.default_rng(605)
    for K in (1, 127, 128, 1000, 1024, 4096):
        codes = np.where(rng.random((7, K)) < 0.5, 1, -1).astype(np.int8)
        packed = torch.full((7, B.bitlinear_packed_row_bytes(K, B1)), 0xAB, dtype=torch.uint8, device="cuda")
        ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        B.bitlinear_pack(dev(codes), B1, packed, ws)
        torch.cuda.synchronize()
        assert B.bitlinear_device_status(ws) == B.BL_OK
        assert np.array_equal(host(packed), orc.pack(codes, B1))


def test_pack_b1_flags_a_zero_code():
    codes = np.ones((2, 64), np.int8)
    codes[1, 5] = 0
    packed = torch.zeros((2, 16), dtype=torch.uint8, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    B.bitlinear_pack(dev(codes), B1, packed, ws)
    assert B.bitlinear_device_status(ws) == B.BL_ERR_BAD_CODE


def check_forward(orc, packed, beta, N, K, x, scale=None, ydts=(B.BL_I32, B.BL_F32, B.BL_BF16)):
    for ydt in ydts:
        y, s = forward(packed, B1, beta, N, K, x, ydt, scale)
        y_ref, s_ref = orc.forward(packed, B1, beta, N, K, x, ydt=ydt, scale=scale)
        assert np.array_equal(s, s_ref)
        if ydt == B.BL_I32:
            assert np.array_equal(y, y_ref)
        elif ydt == B.BL_F32:
            assert_f32_rel(y, y_ref)
        else:
            assert_bf16_ulp(y, y_ref)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 16, 130])
def test_forward_3b_shape(orc, M):
    """3B attention shape (K = 3200: the one-pass prologue for one bf16 token)."""
    N, K = 3200, 3200
    W = synth.normal_f32(610, (N, K), 0.02)
    _, beta, _, packed = binarize(W, codes=False)
    x = synth.to_bf16_bits(synth.normal_f32(611 + M, (M, K)))
    check_forward(orc, packed, beta, N, K, x)


@pytest.mark.parametrize("M,xdt", [(1, "f32"), (1, "i8"), (3, "f32"), (4, "i8"), (7, "f32")])
def test_forward_ragged(orc, M, xdt):
    """K = 1000 (not a multiple of 16: the general prologue), N = 777."""
    N, K = 777, 1000
    W = synth.normal_f32(612, (N, K), 0.02)
    _, beta, _, packed = binarize(W, codes=False)
    x = synth.entry_outliers(synth.normal_f32(613 + M, (M, K)), 614, 0.01, 20.0)
    scale = None
    if xdt == "i8":
        x, scale = orc.act_quant(x)
    check_forward(orc, packed, beta, N, K, x, scale=scale)


def test_forward_70b_down_one_token(orc):
    """70B down-projection shape (K = 28672: 3584-byte rows, the longest the
    1-bit GEMV's planes hold)."""
    N, K = 1024, 28672
    W = synth.normal_f32(615, (N, K), 0.01)
    _, beta, _, packed = binarize(W, codes=False)
    x = synth.to_bf16_bits(synth.normal_f32(616, (1, K)))
    check_forward(orc, packed, beta, N, K, x)


@pytest.mark.parametrize("M", [1, 2])
def test_forward_long_rows_transcoded(orc, M):
    """K = 40000 (5008-byte rows): transcoded to 2 bits in the workspace."""
    N, K = 300, 40000
    W = synth.normal_f32(617, (N, K), 0.01)
    _, beta, _, packed = binarize(W, codes=False)
    x = synth.to_bf16_bits(synth.normal_f32(618 + M, (M, K)))
    check_forward(orc, packed, beta, N, K, x)


def test_forward_many_rows_per_cta(orc):
    """More rows than one CTA's row sums hold (the lean kernel's row tiles)."""
    N, K = 160_000, 128
    W = synth.normal_f32(619, (N, K), 0.02)
    _, beta, _, packed = binarize(W, codes=False)
    x = synth.to_bf16_bits(synth.normal_f32(620, (1, K)))
    check_forward(orc, packed, beta, N, K, x, ydts=(B.BL_I32, B.BL_BF16))


@pytest.mark.parametrize("M", [1, 3, 24])
def test_forward_grouped_b1(orc, M):
    """Three 1-bit layers sharing their input, each with its own beta."""
    K, rows = 1024, [256, 128, 200]
    betas, packs = [], []
    for i, n in enumerate(rows):
        _, b, _, p = binarize(synth.normal_f32(621 + i, (n, K), 0.02 * (i + 1)), codes=False)
        betas.append(b)
        packs.append(p)
    packed = np.concatenate(packs, axis=0)
    x = synth.to_bf16_bits(synth.normal_f32(630 + M, (M, K)))
    N = sum(rows)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(256, B.bitlinear_forward_grouped_workspace_bytes(M, rows, K, B1, B.BL_BF16)),
                     dtype=torch.uint8, device="cuda")
    B.bitlinear_forward_grouped(dev(packed), B1, dev(np.array(betas, np.float32)), rows, K, dev(x), s, y, ws)
    torch.cuda.synchronize()
    assert B.bitlinear_device_status(ws) == B.BL_OK
    yh = host(y)
    off = 0
    for g, n in enumerate(rows):
        y_ref, s_ref = orc.forward(packs[g], B1, betas[g], n, K, x, ydt=0)
        assert np.array_equal(host(s), s_ref)
        assert_f32_rel(yh[:, off:off + n], y_ref)
        off += n


@pytest.mark.parametrize("M", [1, 2])
def test_forward_grouped_b1_long_rows(orc, M):
    """1-bit groups with rows longer than the 1-bit GEMV takes (K = 40000):
    transcoded to 2 bits in the workspace, then the general GEMV kernel with
    the row-group table."""
    K, rows = 40000, [96, 40, 130]
    betas, packs = [], []
    for i, n in enumerate(rows):
        _, b, _, p = binarize(synth.normal_f32(640 + i, (n, K), 0.01 * (i + 1)), codes=False)
        betas.append(b)
        packs.append(p)
    packed = np.concatenate(packs, axis=0)
    x = synth.to_bf16_bits(synth.normal_f32(650 + M, (M, K)))
    N = sum(rows)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.bitlinear_forward_grouped_workspace_bytes(M, rows, K, B1, B.BL_BF16), dtype=torch.uint8,
                     device="cuda")
    B.bitlinear_forward_grouped(dev(packed), B1, dev(np.array(betas, np.float32)), rows, K, dev(x), s, y, ws)
    torch.cuda.synchronize()
    assert B.bitlinear_device_status(ws) == B.BL_OK
    yh = host(y)
    off = 0
    for g, n in enumerate(rows):
        y_ref, s_ref = orc.forward(packs[g], B1, betas[g], n, K, x, ydt=0)
        assert np.array_equal(host(s), s_ref)
        assert_f32_rel(yh[:, off:off + n], y_ref)
        off += n
