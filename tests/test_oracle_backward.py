"""Pins for the oracle's STE backward (CPU only).

The pins: the exact sum of dx checked against Python's ``math.fsum`` (the
correctly rounded fp64 sum of its inputs, which is dx's definition before the
gamma product) on wide-range gradients, hand cases where any fixed fp64 order
loses bits (cancellation, a rounding decided by a far-away term, subnormals),
exact integer arithmetic (integer gradients and a power-of-two gamma make every
sum exact, so the fp32 results equal numpy's int64 products), torch autograd of
the pages' straight-through construction (W_eff = W_q + W - W.detach(), the
same for the activations, gamma held constant) in float64, bf16 gradients
equal to their fp32 widening, and the degenerate cases."""
import math

import numpy as np
import pytest
import torch

from bitlinear_b1_fwd_b200 import synth


def _codes(rng, N, K, p0=0.3):
    u = rng.random((N, K))
    return np.where(u < p0, 0, np.where(u < (1 + p0) / 2, 1, -1)).astype(np.int8)


@pytest.mark.parametrize("M,N,K", [(1, 5, 7), (3, 777, 100), (2, 1000, 33), (1, 64, 16), (1, 65, 16)])
def test_dx_exact_on_integers(orc, M, N, K):
    """Integer dy and gamma = 0.5: the sum is an exact integer and
    dx = 0.5 (dy . W_q) exactly."""
    rng = np.random.default_rng(N)
    codes = _codes(rng, N, K)
    dy = rng.integers(-1000, 1001, size=(M, N)).astype(np.float32)
    dx = orc.backward_dx(codes, dy, 0.5)
    want = (dy.astype(np.int64) @ codes.astype(np.int64)).astype(np.float64) * 0.5
    assert np.array_equal(dx, want.astype(np.float32))


def _fsum_dx(codes, dy, g):
    """dx by its definition with a library routine for the exact sum:
    fp32(gamma * fsum(q dy)), fsum being the correctly rounded fp64 sum."""
    M, N = dy.shape
    K = codes.shape[1]
    out = np.empty((M, K), np.float32)
    for m in range(M):
        for k in range(K):
            terms = [float(dy[m, n]) * int(codes[n, k]) for n in range(N) if codes[n, k]]
            out[m, k] = np.float32(float(np.float32(g)) * math.fsum(terms))
    return out


@pytest.mark.parametrize("g", [1.0, 0.37, 3.0e-3])
def test_dx_is_the_exact_sum_rounded_once(orc, g):
    """Gradients spread over 2^-60 .. 2^60, so every fixed fp64 order loses
    bits somewhere: dx equals fp32(gamma * fsum(q dy)) bit for bit."""
    rng = np.random.default_rng(11)
    M, N, K = 3, 400, 24
    codes = _codes(rng, N, K)
    dy = (rng.standard_normal((M, N)) * np.exp2(rng.integers(-60, 61, size=(M, N)))).astype(np.float32)
    dy[:, ::7] = -np.roll(dy, 1, axis=1)[:, ::7]  # planted cancellations
    assert np.array_equal(orc.backward_dx(codes, dy, g).view(np.uint32), _fsum_dx(codes, dy, g).view(np.uint32))


def test_dx_hand_cases(orc):
    one = np.ones((4, 1), np.int8)
    # cancellation: 1e30 + 1 - 1e30 is 1 exactly (0 in left-to-right fp64)
    dy = np.array([[1e30, 1.0, -1e30, 0.0]], np.float32)
    assert orc.backward_dx(one, dy, 1.0)[0, 0] == 1.0
    # 1 + 2^-24 + 2^-53 + 2^-80: the far term makes fp64 round up, past fp32's tie
    dy = np.array([[1.0, 2.0 ** -24, 2.0 ** -53, 2.0 ** -80]], np.float32)
    assert orc.backward_dx(one, dy, 1.0)[0, 0] == np.float32(1.0 + 2.0 ** -23)
    # without the far term it is an fp32 tie, to even
    dy = np.array([[1.0, 2.0 ** -24, 0.0, 0.0]], np.float32)
    assert orc.backward_dx(one, dy, 1.0)[0, 0] == np.float32(1.0)
    # subnormals add exactly
    tiny = np.float32(2.0 ** -149)
    dy = np.array([[tiny, tiny, tiny, -tiny]], np.float32)
    assert orc.backward_dx(one, dy, 1.0)[0, 0] == np.float32(2.0 ** -148)
    # largest magnitudes: 3 x FLT_MAX - 2 x FLT_MAX, and the sign of -q dy
    big = np.finfo(np.float32).max
    dy = np.array([[big, big, big, 0.0]], np.float32)
    codes = np.array([[1], [1], [-1], [0]], np.int8)
    assert orc.backward_dx(codes, dy, 1.0)[0, 0] == big
    assert orc.backward_dx(codes, -dy, 0.5)[0, 0] == -big / 2


@pytest.mark.parametrize("M,N,K", [(1, 6, 9), (5, 40, 300), (64, 3, 17)])
def test_dw_exact_on_integers(orc, M, N, K):
    """s = 127 makes c = 1: dW = gamma dy^T x_q, exact for integer dy."""
    rng = np.random.default_rng(K)
    dy = rng.integers(-500, 501, size=(M, N)).astype(np.float32)
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    s = np.full(M, 127.0, np.float32)
    dw = orc.backward_dw(dy, xq, s, 0.25)
    want = (dy.astype(np.int64).T @ xq.astype(np.int64)).astype(np.float64) * 0.25
    assert np.array_equal(dw, want.astype(np.float32))


def test_against_autograd_of_the_ste_construction(orc):
    """The pages' BitLinear with straight-through weights and activations:
    out = F.linear(x_deq + x - x.detach(), W_q + W - W.detach()) * gamma, in
    float64 with gamma a constant; autograd's x.grad and W.grad equal the
    oracle's dx and dW up to fp64 summation order (then fp32 rounding)."""
    M, N, K = 6, 300, 200
    Wf = synth.normal_f32(700, (N, K), 0.02)
    xf = synth.normal_f32(701, (M, K))
    g = orc.gamma(Wf)
    codes = orc.ternarize(Wf, g, 1e-5)
    xq, s = orc.act_quant(xf)
    dy = synth.normal_f32(702, (M, N))

    W = torch.tensor(Wf, dtype=torch.float64, requires_grad=True)
    x = torch.tensor(xf, dtype=torch.float64, requires_grad=True)
    Wq = torch.tensor(codes, dtype=torch.float64)
    x_deq = torch.tensor(xq, dtype=torch.float64) * (torch.tensor(s, dtype=torch.float64)[:, None] / 127.0)
    W_eff = Wq + W - W.detach()
    x_ste = x_deq + x - x.detach()
    out = torch.nn.functional.linear(x_ste, W_eff) * float(g)
    (out * torch.tensor(dy, dtype=torch.float64)).sum().backward()

    dx = orc.backward_dx(codes, dy, g).astype(np.float64)
    dw = orc.backward_dw(dy, xq, s, g).astype(np.float64)
    gx = x.grad.numpy()
    gw = W.grad.numpy()
    # fp32 rounding of the same real value: within one fp32 ulp plus fp64 order noise
    bound_x = float(g) * (np.abs(dy).astype(np.float64) @ np.abs(codes).astype(np.float64))
    assert np.all(np.abs(dx - gx) <= 2.0 ** -23 * np.abs(gx) + 1e-12 * bound_x)
    bound_w = float(g) * (np.abs(dy).astype(np.float64).T @ np.abs(x_deq.numpy()))
    assert np.all(np.abs(dw - gw) <= 2.0 ** -23 * np.abs(gw) + 1e-12 * bound_w)
    # and the output itself is the forward's y up to its own rounding
    y, _ = orc.forward(orc.pack(codes, 0), 0, g, N, K, xf, ydt=0)
    assert np.allclose(out.detach().numpy(), y, rtol=1e-5, atol=1e-7)


def test_bf16_gradient_equals_its_widening(orc):
    rng = np.random.default_rng(3)
    codes = _codes(rng, 500, 64)
    dyf = synth.normal_f32(703, (2, 500))
    dyb = synth.to_bf16_bits(dyf)
    dyw = (dyb.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(orc.backward_dx(codes, dyb, 0.37), orc.backward_dx(codes, dyw, 0.37))
    xq, s = orc.act_quant(synth.normal_f32(704, (2, 64)))
    assert np.array_equal(orc.backward_dw(dyb, xq, s, 0.37), orc.backward_dw(dyw, xq, s, 0.37))


def test_degenerate_cases(orc):
    rng = np.random.default_rng(4)
    codes = _codes(rng, 300, 40)
    zero = np.zeros((3, 300), np.float32)
    assert not orc.backward_dx(codes, zero, 0.5).any()
    assert not orc.backward_dx(np.zeros_like(codes), synth.normal_f32(705, (3, 300)), 0.5).any()
    xq, s = orc.act_quant(np.zeros((3, 40), np.float32))  # x_q = 0
    assert not orc.backward_dw(synth.normal_f32(706, (3, 300)), xq, s, 0.5).any()
    # one token, one row: dW is gamma dy x_deq elementwise
    xq, s = orc.act_quant(synth.normal_f32(707, (1, 40)))
    dy = np.array([[1.5]], np.float32)
    dw = orc.backward_dw(dy, xq, s, 2.0)
    want = (2.0 * ((1.5 * xq[0].astype(np.float64)) * (float(s[0]) / 127.0))).astype(np.float32)
    assert np.array_equal(dw[0], want)
