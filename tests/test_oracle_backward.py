"""Pins for the oracle's STE backward (CPU only).

The pins: exact integer arithmetic (integer gradients and a power-of-two gamma
make every sum exact, so the fp32 results equal numpy's int64 products), torch
autograd of the pages' straight-through construction (W_eff = W_q + W -
W.detach(), the same for the activations, gamma held constant) in float64,
bf16 gradients equal to their fp32 widening, and the degenerate cases."""
import numpy as np
import pytest
import torch

from bitlinear_b1_fwd_b200 import synth


def _codes(rng, N, K, p0=0.3):
    u = rng.random((N, K))
    return np.where(u < p0, 0, np.where(u < (1 + p0) / 2, 1, -1)).astype(np.int8)


@pytest.mark.parametrize("M,N,K", [(1, 5, 7), (3, 777, 100), (2, 1000, 33), (1, 64, 16), (1, 65, 16)])
def test_dx_exact_on_integers(orc, M, N, K):
    """Integer dy and gamma = 0.5: every partial sum is an exact integer, so
    the chunk order is immaterial and dx = 0.5 (dy . W_q) exactly."""
    rng = np.random.default_rng(N)
    codes = _codes(rng, N, K)
    dy = rng.integers(-1000, 1001, size=(M, N)).astype(np.float32)
    dx = orc.backward_dx(codes, dy, 0.5)
    want = (dy.astype(np.int64) @ codes.astype(np.int64)).astype(np.float64) * 0.5
    assert np.array_equal(dx, want.astype(np.float32))


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
