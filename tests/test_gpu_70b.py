"""70B-shaped layer (K=8192 -> N=28672 and K=28672 -> N=8192), 2-bit and
base-3 packs, and the token sweep M = 1, 2, 4, ..., 8192 through the forward.

gamma's bits and the packed bytes are compared in full.  For each M the GPU
runs all M tokens; the INT32 accumulators (and the bf16 outputs at a few M)
of every token are checked for M <= 4, and of a seeded sample of tokens plus
the first and last one above that (tokens are independent, so a sample of
rows of y is checked exactly)."""
import numpy as np
import pytest
import torch

from bitlinear_b1_fwd_b200 import binding as B
from bitlinear_b1_fwd_b200 import synth
from gpu_helpers import assert_bf16_ulp

pytestmark = pytest.mark.gpu

I2, T5 = B.BL_PACK_I2, B.BL_PACK_T5
SWEEP = synth.LAYER_70B_M


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bitlinear_b1_fwd_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _sample_rows(M, rng, k=6):
    if M <= 4:
        return np.arange(M)
    rows = set(rng.choice(M, size=min(k, M), replace=False).tolist()) | {0, M - 1}
    return np.array(sorted(rows))


def _oracle_rows(orc, codes, x_rows, g, ydt):
    xq, s = orc.act_quant(np.ascontiguousarray(x_rows))
    acc = orc.matmul_i32(codes, xq, parallel=True)
    return orc.dequant(acc, g, s, ydt), s


@pytest.mark.parametrize("layer", [0, 1])
def test_70b_layer(orc, layer):
    c = synth.LAYER_70B[layer]
    N, K = c["N"], c["K"]
    W = synth.layer_70b_weights(layer)
    g_ref = orc.gamma(W)
    codes = orc.ternarize(W, g_ref, 1e-5, parallel=True)
    Wd = torch.from_numpy(W).cuda()
    del W
    x_all = synth.layer_70b_acts(layer, SWEEP[-1])
    xd_all = torch.from_numpy(x_all.view(np.int16)).cuda().view(torch.bfloat16)
    rng = np.random.default_rng(700 + layer)
    for fmt in (I2, T5):
        rb = B.bitlinear_packed_row_bytes(K, fmt)
        packed = torch.empty((N, rb), dtype=torch.uint8, device="cuda")
        gamma = torch.empty(1, dtype=torch.float32, device="cuda")
        ws = torch.zeros(B.bitlinear_quantize_weights_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
        B.bitlinear_quantize_weights(Wd, 1e-5, fmt, packed, None, gamma, ws)
        torch.cuda.synchronize()
        assert B.bitlinear_device_status(ws) == B.BL_OK
        assert np.float32(gamma.item()).view(np.uint32) == g_ref.view(np.uint32)
        assert np.array_equal(packed.cpu().numpy(), orc.pack(codes, fmt))
        for M in SWEEP:
            xd = xd_all[:M]
            ydts = (B.BL_I32, B.BL_BF16) if M in (1, 4, 64, 8192) else (B.BL_I32,)
            for ydt in ydts:
                tdt = torch.int32 if ydt == B.BL_I32 else torch.bfloat16
                y = torch.empty((M, N), dtype=tdt, device="cuda")
                scale = torch.empty(M, dtype=torch.float32, device="cuda")
                fws = torch.zeros(B.bitlinear_forward_workspace_bytes(M, N, K, fmt, B.BL_BF16),
                                  dtype=torch.uint8, device="cuda")
                B.bitlinear_forward(packed, fmt, gamma, N, K, xd, scale, y, fws)
                torch.cuda.synchronize()
                assert B.bitlinear_device_status(fws) == B.BL_OK
                rows = _sample_rows(M, rng)
                idx = torch.from_numpy(rows).cuda()
                got = y.index_select(0, idx)
                got = got.view(torch.int16).cpu().numpy().view(np.uint16) if ydt == B.BL_BF16 else got.cpu().numpy()
                ref, s_ref = _oracle_rows(orc, codes, x_all[rows], g_ref, ydt)
                assert np.array_equal(scale.index_select(0, idx).cpu().numpy(), s_ref)
                if ydt == B.BL_I32:
                    assert np.array_equal(got, ref), (fmt, M)
                else:
                    assert_bf16_ulp(got, ref)
                del y, fws
        del packed
