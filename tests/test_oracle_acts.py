"""Pins for the oracle's per-token absmax INT8 quantization (CPU only)."""
import numpy as np
import pytest

from bitlinear_b1_fwd_b200 import synth


def _tie_input(target):
    """An fp32 x in (0, 1) with fl32(fl32(x / 1) * 127) == target exactly
    (searched with numpy's IEEE fp32 multiply)."""
    v = np.float32(target / 127.0)
    for _ in range(400):
        t = np.float32(v * np.float32(127.0))
        if t == np.float32(target):
            return v
        v = np.nextafter(v, np.float32(1) if t < target else np.float32(0))
    raise AssertionError(f"no fp32 input reaches {target}")


def test_round_half_to_even(orc):
    """A token whose largest |x| is 1.0 (so x / s is exact) with entries that
    land exactly on k + 0.5 after the multiply by 127: half-to-even gives
    0.5 -> 0, 1.5 -> 2, 2.5 -> 2, 3.5 -> 4, -2.5 -> -2, 126.5 -> 126."""
    ties = {0.5: 0, 1.5: 2, 2.5: 2, 3.5: 4, 126.5: 126}
    xs = [np.float32(1.0)]
    want = [127]
    for t, q in ties.items():
        v = _tie_input(t)
        xs += [v, -v]
        want += [q, -q]
    x = np.array([xs], np.float32)
    xq, s = orc.act_quant(x)
    assert s[0] == np.float32(1.0)
    assert xq[0].tolist() == want


def test_hand_row(orc):
    """x = [1, -0.5, 0.25, 0, 2]: s = 2, x/s*127 = [63.5, -31.75, 15.875, 0, 127]
    -> [64, -32, 16, 0, 127]."""
    xq, s = orc.act_quant(np.array([[1.0, -0.5, 0.25, 0.0, 2.0]], np.float32))
    assert s.tolist() == [2.0]
    assert xq[0].tolist() == [64, -32, 16, 0, 127]


def test_invariants_random(orc):
    x = synth.entry_outliers(synth.normal_f32(2001, (64, 999)), 3001, 0.01, 20.0)
    xq, s = orc.act_quant(x)
    assert xq.min() >= -127 and xq.max() <= 127            # symmetric, never -128
    assert np.array_equal(s, np.abs(x).max(axis=1))         # per-token absmax
    # the entry holding max|x| maps to exactly +-127 (x/s = +-1 exactly)
    am = np.abs(x).argmax(axis=1)
    assert np.array_equal(np.abs(xq[np.arange(64), am]), np.full(64, 127, np.int8))
    # sign symmetry and invariance under power-of-two rescaling
    xq2, s2 = orc.act_quant(-x)
    assert np.array_equal(xq2, -xq) and np.array_equal(s2, s)
    xq3, s3 = orc.act_quant(x * np.float32(0.125))
    assert np.array_equal(xq3, xq) and np.array_equal(s3, s * np.float32(0.125))
    # error bound of a symmetric absmax grid: |x - x_q * s / 127| <= s / 254 (+ rounding)
    err = np.abs(x.astype(np.float64) - xq.astype(np.float64) * s[:, None] / 127.0)
    assert (err <= s[:, None].astype(np.float64) / 254.0 * (1 + 1e-5)).all()


def test_zero_and_tiny_rows(orc):
    """A zero token has scale 1e-6 (the floor) and codes 0; a token below the
    floor is quantized against the floor, not its own max."""
    x = np.zeros((3, 7), np.float32)
    x[1, 2] = 5e-7
    x[2, :] = np.float32(1e-3)
    xq, s = orc.act_quant(x)
    assert s[0] == np.float32(1e-6) and not xq[0].any()
    assert s[1] == np.float32(1e-6)
    assert xq[1, 2] == np.rint(np.float32(np.float32(5e-7) / np.float32(1e-6)) * np.float32(127))
    assert (xq[2] == 127).all()


def test_bf16_input_same_as_widened(orc):
    x = synth.normal_f32(77, (5, 3200))
    xb = synth.to_bf16_bits(x)
    a = orc.act_quant(xb)
    b = orc.act_quant(synth.bf16_bits_to_f32(xb))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_matches_pages_torch_function(orc):
    """Cross-check only (the same formula run by torch's CPU ops, as the page's
    activation_quantize_int8 writes it)."""
    import torch
    x = synth.normal_f32(78, (16, 513))
    t = torch.from_numpy(x)
    scale = t.abs().amax(dim=-1, keepdim=True).clamp(min=1e-6)
    ref = torch.clamp(torch.round(t / scale * 127), -127, 127).to(torch.int8).numpy()
    xq, s = orc.act_quant(x)
    assert np.array_equal(xq, ref)
    assert np.array_equal(s, scale[:, 0].numpy())


def _division_sensitive_rows(count=64):
    """Tokens in which x / s * 127 (the page's order) and x * (1 / s) * 127
    round to different integers for at least one entry."""
    rows = []
    seed = 500
    while len(rows) < count:
        x = synth.normal_f32(seed, (256, 64))
        seed += 1
        s = np.abs(x).max(axis=1, keepdims=True)
        a = np.rint((x / s) * np.float32(127))
        b = np.rint((x * (np.float32(1) / s)) * np.float32(127))
        for i in np.nonzero((a != b).any(axis=1))[0]:
            rows.append(x[i])
    return np.array(rows[:count], np.float32)


def test_division_not_reciprocal(orc):
    """The page divides by the scale before multiplying by 127.  On tokens
    where a reciprocal-multiply would round differently, the oracle must agree
    with the page's expression as torch evaluates it."""
    import torch
    x = _division_sensitive_rows()
    t = torch.from_numpy(x)
    scale = t.abs().amax(dim=-1, keepdim=True).clamp(min=1e-6)
    ref = torch.clamp(torch.round(t / scale * 127), -127, 127).to(torch.int8).numpy()
    recip = torch.clamp(torch.round(t * (1.0 / scale) * 127), -127, 127).to(torch.int8).numpy()
    assert not np.array_equal(ref, recip)
    xq, _ = orc.act_quant(x)
    assert np.array_equal(xq, ref)
