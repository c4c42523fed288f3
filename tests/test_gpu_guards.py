"""Out-of-bounds writes: every output array and workspace of a call sits
between two 4 KB guard regions filled with 0xA5, on odd tiny shapes (K = 5, 7,
129; M = 1..17; N not a multiple of any tile) and the workspace exactly the
queried size; after the call the guards must be intact and the outputs equal
the oracle's."""
import numpy as np
import pytest
import torch

from bitlinear_b1_fwd_b200 import binding as B
from bitlinear_b1_fwd_b200 import synth
from gpu_helpers import assert_bf16_ulp, assert_f32_rel, dev, host

pytestmark = pytest.mark.gpu

G = 4096
I2, T5, B1 = B.BL_PACK_I2, B.BL_PACK_T5, B.BL_PACK_B1


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bitlinear_b1_fwd_b200 import build
    build.build()
    assert torch.cuda.is_available()
    torch.cuda.init()


class Guarded:
    """A device array of `shape` and `dtype` between two guard regions."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = n
        self.buf = torch.full((G + n + G,), 0xA5, dtype=torch.uint8, device="cuda")
        self.t = self.buf[G:G + n].view(dtype).view(shape) if n else torch.empty(shape, dtype=dtype, device="cuda")

    def intact(self):
        b = host(self.buf)
        return bool((b[:G] == 0xA5).all() and (b[G + self.nbytes:] == 0xA5).all())


def ws_guarded(nbytes):
    w = Guarded((max(int(nbytes), B.BL_WS_HEADER_BYTES),), torch.uint8)
    w.t.zero_()
    return w


def check_intact(*gs):
    torch.cuda.synchronize()
    for i, g in enumerate(gs):
        assert g.intact(), f"guard {i} overwritten"


@pytest.mark.parametrize("N,K,fmt", [(7, 5, I2), (13, 129, T5), (130, 7, I2), (33, 129, I2)])
def test_quantize_weights(orc, N, K, fmt):
    W = synth.normal_f32(800 + K, (N, K), 0.02)
    rb = B.bitlinear_packed_row_bytes(K, fmt)
    packed, codes, gamma = Guarded((N, rb), torch.uint8), Guarded((N, K), torch.int8), Guarded((1,), torch.float32)
    ws = ws_guarded(B.bitlinear_quantize_weights_workspace_bytes(N, K))
    B.bitlinear_quantize_weights(dev(W), 1e-5, fmt, packed.t, codes.t, gamma.t, ws.t)
    check_intact(packed, codes, gamma, ws)
    g = orc.gamma(W)
    assert host(gamma.t)[0] == g
    assert np.array_equal(host(codes.t), orc.ternarize(W, g, 1e-5))
    assert np.array_equal(host(packed.t), orc.pack(host(codes.t), fmt))


@pytest.mark.parametrize("N,K", [(7, 5), (13, 129), (3, 300)])
def test_binarize_weights(orc, N, K):
    W = synth.normal_f32(810 + K, (N, K), 0.02)
    rb = B.bitlinear_packed_row_bytes(K, B1)
    packed, codes = Guarded((N, rb), torch.uint8), Guarded((N, K), torch.int8)
    beta, alpha = Guarded((1,), torch.float32), Guarded((1,), torch.float32)
    ws = ws_guarded(B.bitlinear_binarize_weights_workspace_bytes(N, K))
    B.bitlinear_binarize_weights(dev(W), packed.t, codes.t, beta.t, alpha.t, ws.t)
    check_intact(packed, codes, beta, alpha, ws)
    a, b, c = orc.binarize_weights(W)
    assert host(alpha.t)[0] == a and host(beta.t)[0] == b
    assert np.array_equal(host(codes.t), c)
    assert np.array_equal(host(packed.t), orc.pack(c, B1))


@pytest.mark.parametrize("M,K", [(17, 129), (3, 5), (1, 7)])
def test_quantize_acts_and_layernorm(orc, M, K):
    x = synth.normal_f32(820 + K, (M, K))
    xq, s = Guarded((M, K), torch.int8), Guarded((M,), torch.float32)
    B.bitlinear_quantize_acts(dev(x), xq.t, s.t)
    check_intact(xq, s)
    xq_ref, s_ref = orc.act_quant(x)
    assert np.array_equal(host(xq.t), xq_ref) and np.array_equal(host(s.t), s_ref)
    g, b = synth.normal_f32(821, (K,), 1.0), synth.normal_f32(822, (K,), 0.1)
    y, xq2, s2 = Guarded((M, K), torch.int16), Guarded((M, K), torch.int8), Guarded((M,), torch.float32)
    B.bitlinear_layernorm_quantize_acts(dev(x), dev(g), dev(b), 1e-5, xq2.t, s2.t, y.t)
    check_intact(y, xq2, s2)
    y_ref, xq_ref, s_ref = orc.layernorm_quant(x, g, b, 1e-5)
    assert np.array_equal(host(y.t).view(np.uint16), y_ref)
    assert np.array_equal(host(xq2.t), xq_ref) and np.array_equal(host(s2.t), s_ref)


def _packed(orc, N, K, fmt, seed):
    W = synth.normal_f32(seed, (N, K), 0.02)
    if fmt == B1:
        _, beta, codes = orc.binarize_weights(W)
        return np.float32(beta), orc.pack(codes, B1)
    g = orc.gamma(W)
    return g, orc.pack(orc.ternarize(W, g, 1e-5), fmt)


@pytest.mark.parametrize("M,N,K,fmt", [(1, 13, 129, I2), (3, 130, 7, T5), (5, 13, 5, B1), (17, 33, 129, I2),
                                       (17, 130, 256, I2), (9, 200, 512, T5), (6, 131, 384, B1)])
def test_forward(orc, M, N, K, fmt):
    g, packed = _packed(orc, N, K, fmt, 830 + N)
    x = synth.to_bf16_bits(synth.normal_f32(831 + M, (M, K)))
    for ydt, tdt in ((B.BL_F32, torch.float32), (B.BL_BF16, torch.bfloat16), (B.BL_I32, torch.int32)):
        y, s = Guarded((M, N), tdt), Guarded((M,), torch.float32)
        ws = ws_guarded(B.bitlinear_forward_workspace_bytes(M, N, K, fmt, B.BL_BF16))
        B.bitlinear_forward(dev(packed), fmt, dev(np.array([g], np.float32)), N, K, dev(x), s.t, y.t, ws.t)
        check_intact(y, s, ws)
        assert B.bitlinear_device_status(ws.t) == B.BL_OK
        y_ref, s_ref = orc.forward(packed, fmt, g, N, K, x, ydt=ydt)
        assert np.array_equal(host(s.t), s_ref)
        got = host(y.t)
        if ydt == B.BL_BF16:
            assert_bf16_ulp(got, y_ref)
        elif ydt == B.BL_F32:
            assert_f32_rel(got, y_ref)
        else:
            assert np.array_equal(got, y_ref)


@pytest.mark.parametrize("M", [1, 6])
def test_forward_grouped(orc, M):
    K, rows = 256, [13, 7, 33]
    parts = [_packed(orc, n, K, I2, 840 + i) for i, n in enumerate(rows)]
    packed = np.concatenate([p for _, p in parts], axis=0)
    gammas = np.array([g for g, _ in parts], np.float32)
    x = synth.normal_f32(845 + M, (M, K))
    N = sum(rows)
    y, s = Guarded((M, N), torch.float32), Guarded((M,), torch.float32)
    ws = ws_guarded(B.bitlinear_forward_grouped_workspace_bytes(M, rows, K, I2, B.BL_F32))
    B.bitlinear_forward_grouped(dev(packed), I2, dev(gammas), rows, K, dev(x), s.t, y.t, ws.t)
    check_intact(y, s, ws)
    off = 0
    for (g, p), n in zip(parts, rows):
        y_ref, _ = orc.forward(p, I2, g, n, K, x, ydt=B.BL_F32)
        assert_f32_rel(host(y.t)[:, off:off + n], y_ref)
        off += n


@pytest.mark.parametrize("M,N,K", [(1, 13, 129), (3, 130, 7), (5, 65, 33)])
def test_backward(orc, M, N, K):
    g, packed = _packed(orc, N, K, I2, 850 + K)
    codes = orc.unpack(packed, N, K, I2)
    dy = synth.normal_f32(851, (M, N), 1e-2)
    dx = Guarded((M, K), torch.float32)
    ws = ws_guarded(B.bitlinear_backward_dx_workspace_bytes(M, N, K, I2))
    B.bitlinear_backward_dx(dev(packed), I2, dev(np.array([g], np.float32)), N, K, dev(dy), dx.t, ws.t)
    check_intact(dx, ws)
    assert np.array_equal(host(dx.t), orc.backward_dx(codes, dy, g))
    xq, s = orc.act_quant(synth.normal_f32(852, (M, K)))
    dw = Guarded((N, K), torch.float32)
    B.bitlinear_backward_dw(dev(dy), dev(xq), dev(s), dev(np.array([g], np.float32)), dw.t)
    check_intact(dw)
    assert np.array_equal(host(dw.t), orc.backward_dw(dy, xq, s, g))
