"""Seeded synthetic inputs for the BitLinear forward.

This module only draws numbers: it holds none of the method's arithmetic, so
both the CUDA path (through ``bench.py`` and the tests) and the CPU oracle can
be fed from it.

Recipe: a counter-based splitmix64 stream (state_i = seed + i * 0x9E3779B97F4A7C15,
standard splitmix64 output mix), 53-bit uniforms, Box-Muller in fp64, rounded
to fp32; bf16 activations are the round-to-nearest-even bf16 of those fp32
values (torch's conversion).  Shapes follow LLaMA-style linear layers of a
3B and a 70B model; weights are N(0, 0.02) (3B) or N(0, 0.01) (70B) latent
fp32 matrices, activations N(0, 1), with the outlier patterns listed per
workload.
"""
from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_BLOCK = 1 << 22


def splitmix64(seed: int, start: int, n: int) -> np.ndarray:
    """Outputs start..start+n-1 of the splitmix64 stream for ``seed``."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def uniform(seed: int, n: int) -> np.ndarray:
    """n uniforms in [0, 1) (fp64, 53 random bits each)."""
    z = splitmix64(seed, 0, n)
    return (z >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal_f32(seed: int, shape, sigma: float = 1.0) -> np.ndarray:
    """N(0, sigma^2) samples rounded to fp32, generated block by block."""
    n = int(np.prod(shape))
    out = np.empty(n, np.float32)
    npairs = (n + 1) // 2
    for p0 in range(0, npairs, _BLOCK):
        cnt = min(_BLOCK, npairs - p0)
        z = splitmix64(seed, 2 * p0, 2 * cnt)
        u1 = ((z[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
        u2 = (z[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
        r = np.sqrt(-2.0 * np.log(u1)) * sigma
        th = 2.0 * np.pi * u2
        blk = np.empty(2 * cnt, np.float64)
        blk[0::2] = r * np.cos(th)
        blk[1::2] = r * np.sin(th)
        lo = 2 * p0
        hi = min(n, lo + 2 * cnt)
        out[lo:hi] = blk[: hi - lo].astype(np.float32)
    return out.reshape(shape)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """bf16 (round to nearest even, by torch) of an fp32 array, as uint16 bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def entry_outliers(x: np.ndarray, seed: int, p: float, factor: float) -> np.ndarray:
    """Scale each entry independently by ``factor`` with probability ``p``."""
    mask = uniform(seed, x.size).reshape(x.shape) < p
    y = x.copy()
    y[mask] *= np.float32(factor)
    return y


def channel_outliers(x: np.ndarray, seed: int, count: int, factor: float) -> np.ndarray:
    """Scale ``count`` seeded input channels (columns) by ``factor`` for every token."""
    K = x.shape[-1]
    ch = np.argsort(uniform(seed, K), kind="stable")[:count]
    y = x.copy()
    y[..., ch] *= np.float32(factor)
    return y


# ----------------------------------------------------------------------------
# Workloads.  Seeds: weights 1000 + w, activations 2000 + w, outlier masks
# 3000 + w, where w numbers the workload (layer index added in hundreds).
# ----------------------------------------------------------------------------

TINY = dict(name="tiny", M=8, K=256, N=512, w_sigma=0.02)
DECODE_3B = [dict(name="3b_up", M=1, K=3200, N=8640, w_sigma=0.02),
             dict(name="3b_down", M=1, K=8640, N=3200, w_sigma=0.02)]
PREFILL_3B = dict(name="3b_prefill", M=4096, K=3200, N=8640, w_sigma=0.02)
BLOCK_3B = [dict(name="q", K=3200, N=3200), dict(name="k", K=3200, N=3200),
            dict(name="v", K=3200, N=3200), dict(name="o", K=3200, N=3200),
            dict(name="up", K=3200, N=8640), dict(name="down", K=8640, N=3200)]
BLOCK_3B_M = (1, 16, 128, 1024)
LAYER_70B = [dict(name="70b_up", K=8192, N=28672, w_sigma=0.01),
             dict(name="70b_down", K=28672, N=8192, w_sigma=0.01)]
LAYER_70B_M = tuple(2 ** i for i in range(14))  # 1, 2, 4, ..., 8192

# The pages' two five-weight worked examples, as 1 x 5 weight matrices.
EXAMPLE_A = np.array([[0.20, -0.90, 1.30, -0.60, 0.05]], np.float32)
EXAMPLE_B = np.array([[0.9, -0.3, 0.05, -1.2, 0.4]], np.float32)


def tiny_inputs():
    """Tiny BitLinear: W fp32 [512, 256] N(0, 0.02); x fp32 [8, 256] N(0, 1)
    with each entry x20 with probability 0.01."""
    W = normal_f32(1001, (512, 256), 0.02)
    x = entry_outliers(normal_f32(2001, (8, 256)), 3001, 0.01, 20.0)
    return W, x


def decode_3b_inputs(layer: int):
    """3B decode GEMV, layer 0 = up (K 3200 -> N 8640), 1 = down (8640 -> 3200):
    W fp32 N(0, 0.02), x one bf16 token N(0, 1)."""
    c = DECODE_3B[layer]
    W = normal_f32(1002 + 100 * layer, (c["N"], c["K"]), c["w_sigma"])
    x = to_bf16_bits(normal_f32(2002 + 100 * layer, (c["M"], c["K"])))
    return W, x


def prefill_3b_inputs(M: int | None = None):
    """3B prefill: W fp32 [8640, 3200] N(0, 0.02); x bf16 [4096, 3200] N(0, 1)
    with 16 of the 3200 channels (0.5 %) x30 for every token.  ``M`` < 4096
    gives the first M tokens of the same stream."""
    c = PREFILL_3B
    M = c["M"] if M is None else M
    W = normal_f32(1003, (c["N"], c["K"]), c["w_sigma"])
    x = normal_f32(2003, (M, c["K"]))
    x = channel_outliers(x, 3003, 16, 30.0)
    return W, to_bf16_bits(x)


def block_3b_inputs(layer: int, M: int):
    c = BLOCK_3B[layer]
    W = normal_f32(1004 + 100 * layer, (c["N"], c["K"]), 0.02)
    x = to_bf16_bits(normal_f32(2004 + 100 * layer, (M, c["K"])))
    return W, x


def layer_70b_weights(layer: int):
    c = LAYER_70B[layer]
    return normal_f32(1005 + 100 * layer, (c["N"], c["K"]), c["w_sigma"])


def layer_70b_acts(layer: int, M: int):
    c = LAYER_70B[layer]
    return to_bf16_bits(normal_f32(2005 + 100 * layer, (M, c["K"])))
