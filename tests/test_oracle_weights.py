"""Pins for the oracle's absmean scale and ternarization (CPU only).

Each check rests on something other than the oracle itself: the pages' worked
examples (tests/golden), the threshold form the pages state, exact rational
arithmetic, or closed-form statistics of a Gaussian.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from conftest import read_golden
from bitlinear_b1_fwd_b200 import synth


# --- worked examples ------------------------------------------------------

def test_worked_example_a(orc):
    g = read_golden("worked_example_a.txt")
    W = np.array([[float(v) for v in g["W"]]], np.float32)
    gamma = orc.gamma(W)
    assert round(float(gamma), 2) == float(g["gamma"][0])
    # the page divides by gamma and prints two decimals
    wn = W.astype(np.float64) / float(gamma)
    assert [round(v, 2) for v in wn[0]] == [float(v) for v in g["W_norm"]]
    codes = orc.ternarize(W, gamma, 1e-5)
    assert codes[0].tolist() == [int(v) for v in g["W_q"]]


def test_worked_example_b_ternary_and_onebit(orc):
    g = read_golden("worked_example_b.txt")
    w = np.array([float(v) for v in g["w"]], np.float32)
    gamma = orc.gamma(w[None, :])
    assert round(float(gamma), 2) == float(g["gamma"][0])
    q = orc.ternarize(w[None, :], gamma, 1e-5)[0]
    b, alpha, beta = orc.onebit(w)
    assert round(float(beta), 2) == float(g["beta"][0])
    i = int(g["onebit_err_idx"][0])
    # 1-bit sends the small weight to +beta, error 0.52
    assert b[i] == 1
    assert round(abs(float(beta) * b[i] - float(w[i])), 2) == float(g["onebit_err"][0])
    # ternary sends it to 0, error 0.05
    assert q[i] == 0
    assert round(abs(float(gamma) * q[i] - float(w[i])), 2) == float(g["ternary_err"][0])
    # the other four weights come out the same in both versions
    for j in (int(v) for v in g["unchanged_idx"]):
        assert q[j] * float(gamma) == pytest.approx(b[j] * float(beta), abs=1e-6)
    # alpha is the plain mean; the 1-bit signs are the centred ones
    assert float(alpha) == pytest.approx(-0.03, abs=1e-6)
    assert b.tolist() == [1, -1, 1, -1, 1]


# --- threshold form -------------------------------------------------------

def _fp32_div_is_half(w, d):
    """True iff fl32(|w| / d) == 0.5 while |w| / d > 0.5 exactly (the only way
    the divide-and-round form can differ from the threshold form)."""
    r = Fraction(abs(float(w))) / Fraction(float(d))
    return r > Fraction(1, 2) and np.float32(abs(np.float32(w)) / np.float32(d)) == np.float32(0.5)


@pytest.mark.parametrize("seed", [11, 12])
def test_threshold_form(orc, seed):
    """|w| <= gamma/2 -> 0; w > gamma/2 -> +1; w < -gamma/2 -> -1, evaluated in
    exact arithmetic against d = gamma + eps.  The two forms agree on every fp32
    weight: d/2 is exact, and the next fp32 above it is d/2 (1 + 2^-23 / m)
    (m < 2 the significand of d), whose quotient by d exceeds the rounding
    midpoint 1/2 + 2^-25, so no quotient above 1/2 rounds down to 1/2."""
    W = synth.normal_f32(seed, (64, 1000), 0.02)
    gamma = orc.gamma(W)
    d = np.float32(gamma + np.float32(1e-5))
    # plant weights right at and around the boundary d/2
    half = np.float32(d / np.float32(2))
    plant = [half, -half, np.nextafter(half, np.float32(1)), np.nextafter(half, np.float32(0)),
             -np.nextafter(half, np.float32(1)), np.float32(0), np.float32(-0.0),
             np.float32(3 * half), np.float32(d)]
    W[0, :len(plant)] = plant
    codes = orc.ternarize(W, gamma, 1e-5)
    two_abs = 2.0 * np.abs(W.astype(np.float64))      # exact in fp64
    dd = float(d)
    expect = np.where(two_abs <= dd, 0, np.sign(W)).astype(np.int8)
    diff = np.argwhere(codes != expect)
    assert len(diff) == 0, [(n, k, W[n, k], _fp32_div_is_half(W[n, k], d)) for (n, k) in diff[:5]]
    assert set(np.unique(codes).tolist()) <= {-1, 0, 1}
    assert codes[0, 0] == 0 and codes[0, 1] == 0     # exactly gamma/2 -> 0 (half-to-even)


def test_threshold_form_over_many_scales(orc):
    """The threshold form at the boundary d/2 for 512 scales spread over three
    binades: the weights d/2, its fp32 neighbours and their negatives.  A
    quotient taken as w * fl(1/d) instead of one division disagrees with the
    threshold on about a fifth of the scales (fl(1/d) carries up to half an
    ulp of error, enough to move w = d/2 -+ 1 ulp across 1/2)."""
    gammas = (0.0025 + 0.0175 * synth.uniform(17, 512)).astype(np.float32)
    eps = np.float32(1e-5)
    for gamma in gammas:
        d = np.float32(gamma + eps)
        half = np.float32(d / np.float32(2))
        up, down = np.nextafter(half, np.float32(1)), np.nextafter(half, np.float32(0))
        W = np.array([[half, up, down, -half, -up, -down]], np.float32)
        codes = orc.ternarize(W, np.float32(gamma), 1e-5)[0]
        assert codes.tolist() == [0, 1, 0, 0, -1, 0], (float(gamma), codes.tolist())


# --- exact value of gamma ---------------------------------------------------

def _exact_abs_sum(W):
    """Exact sum of |w| over fp32 W as an integer multiple of 2^-149."""
    bits = np.abs(W).astype(np.float32).view(np.uint32).ravel()
    e = (bits >> 23).astype(np.int64)
    m = (bits & 0x7FFFFF).astype(np.int64)
    mant = np.where(e > 0, m | 0x800000, m)
    shift = np.maximum(e, 1) - 1
    total = 0
    for s in np.unique(shift):
        total += int(mant[shift == s].sum()) << int(s)
    return total


def _round_fraction_to_f32(fr):
    """Round a positive Fraction to the nearest fp32 (ties to even)."""
    c = np.float32(float(fr))
    best = None
    for cand in (np.nextafter(c, np.float32(0)), c, np.nextafter(c, np.float32(np.inf))):
        err = abs(Fraction(float(cand)) - fr)
        key = (err, int(np.float32(cand).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return best[1]


@pytest.mark.parametrize("shape,sigma,seed", [((512, 256), 0.02, 1001), ((3, 5), 1.0, 5),
                                              ((37, 1111), 0.01, 7), ((1, 8193), 0.5, 8)])
def test_gamma_matches_exact_sum(orc, shape, sigma, seed):
    W = synth.normal_f32(seed, shape, sigma)
    T = W.size
    exact = Fraction(_exact_abs_sum(W), 2 ** 149)
    S = orc.absmean_sum(W)
    # fp64 summation error bound: (terms per lane + tree depth) * eps * sum
    depth = 32 + 8 + math.ceil(math.log2(max(2, T / 8192))) + 1
    assert abs(Fraction(S) - exact) <= depth * Fraction(2) ** -53 * exact
    gamma = orc.gamma(W)
    want = _round_fraction_to_f32(exact / T)
    assert abs(int(np.float32(gamma).view(np.int32)) - int(np.float32(want).view(np.int32))) <= 1
    assert gamma == want   # equal unless gamma64 falls within ~1e-16 of a rounding midpoint


def test_gamma_bf16_input(orc):
    """bf16 latent weights are widened exactly: gamma equals the gamma of the
    same values held in fp32."""
    W = synth.normal_f32(21, (40, 300), 0.02)
    Wb = synth.to_bf16_bits(W)
    Wf = synth.bf16_bits_to_f32(Wb)
    assert orc.gamma(Wb) == orc.gamma(Wf)
    assert np.array_equal(orc.ternarize(Wb, orc.gamma(Wb)), orc.ternarize(Wf, orc.gamma(Wf)))


# --- closed-form statistics of Gaussian weights ------------------------------

def test_gaussian_statistics(orc):
    """For W ~ N(0, s^2): gamma -> s * sqrt(2/pi); P(code 0) -> P(|z| <= sqrt(2/pi)/2)
    = erf(1 / (2 sqrt(pi))) = 0.3101; P(+1) = P(-1)."""
    s = 0.02
    W = synth.normal_f32(31, (1024, 2048), s)
    gamma = float(orc.gamma(W))
    assert gamma == pytest.approx(s * math.sqrt(2 / math.pi), rel=2e-3)
    codes = orc.ternarize(W, gamma, 1e-5)
    p0 = float(np.mean(codes == 0))
    want0 = math.erf(1.0 / (2.0 * math.sqrt(math.pi)))
    assert want0 == pytest.approx(0.3101, abs=1e-4)
    assert p0 == pytest.approx(want0, abs=3e-3)
    pp, pm = float(np.mean(codes == 1)), float(np.mean(codes == -1))
    assert pp == pytest.approx(pm, abs=3e-3)


def test_degenerate_weights(orc):
    """All-zero W: gamma 0, d = eps, every code 0.  A constant matrix c: gamma = |c|,
    every ratio is c/(|c|+eps) -> +-1."""
    Z = np.zeros((3, 17), np.float32)
    assert orc.gamma(Z) == 0.0
    assert not orc.ternarize(Z, 0.0).any()
    Cm = np.full((2, 9), -0.75, np.float32)
    assert orc.gamma(Cm) == np.float32(0.75)
    assert (orc.ternarize(Cm, orc.gamma(Cm)) == -1).all()
    # a single huge weight: gamma = w/T, the big weight clamps to 1, the rest to 0
    W = np.zeros((1, 100), np.float32)
    W[0, 3] = 1000.0
    g = orc.gamma(W)
    assert g == np.float32(10.0)
    c = orc.ternarize(W, g)
    assert c[0, 3] == 1 and np.count_nonzero(c) == 1


def test_onebit_centring(orc):
    """1-bit weights compare against the mean alpha, not against zero: for
    w = [0.01, 0.5, 0.6, 0.7] the mean is 0.4525, so the small positive weight
    maps to -1; beta is the mean |w| = 0.4525 as well."""
    b, alpha, beta = orc.onebit(np.array([0.01, 0.5, 0.6, 0.7], np.float32))
    assert b.tolist() == [-1, 1, 1, 1]
    assert float(alpha) == pytest.approx(0.4525, abs=1e-6)
    assert float(beta) == pytest.approx(0.4525, abs=1e-6)
    b, alpha, beta = orc.onebit(np.array([-0.4, -0.1, 0.2, -0.5], np.float32))
    assert b.tolist() == [-1, 1, 1, -1]                     # alpha = -0.2
    assert float(beta) == pytest.approx(0.3, abs=1e-6)
