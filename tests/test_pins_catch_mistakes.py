"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of the oracle's C source (a dropped
term, a wrong factor, a reversed index or bit order, a different rounding or
tie rule, a missing tree level), builds the copy with the oracle's own gcc
flags, and runs the oracle pin tests (``tests/test_oracle_*.py``) against it
in a child process: at least one pin must fail for every planted mistake.
The unchanged oracle passes the same pins in the main run."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "bitlinear_oracle.c")
PIN_FILES = sorted(os.path.join(ROOT, "tests", f) for f in os.listdir(os.path.join(ROOT, "tests"))
                   if f.startswith("test_oracle_") and f.endswith(".py"))

# (name, text in the source, replacement): each text occurs exactly once
MISTAKES = [
    ("gamma_divides_by_N", "double g = S / (double)(N * K);", "double g = S / (double)N;"),
    ("gamma_without_abs", "acc += (double)(absval ? fabsf(w) : w);", "acc += (double)w;"),
    ("gamma_tree_drops_a_level", "for (int64_t s = P / 2; s >= 1; s /= 2)", "for (int64_t s = P / 2; s >= 2; s /= 2)"),
    ("ternarize_without_eps", "float d = gamma + eps;", "float d = gamma;"),
    ("ternarize_rounds_half_away", "float q = nearbyintf(r);", "float q = roundf(r);"),
    ("pack_digits_reversed", "byte |= digit << (2 * i);", "byte |= digit << (6 - 2 * i);"),
    ("act_quant_times_128", "t = t * 127.0f;", "t = t * 128.0f;"),
    ("act_quant_without_floor", "float s = amax > 1e-6f ? amax : 1e-6f;", "float s = amax;"),
    ("matmul_k_reversed", "s += (int32_t)codes[n * K + k] * (int32_t)xq[m * K + k];",
     "s += (int32_t)codes[n * K + k] * (int32_t)xq[m * K + (K - 1 - k)];"),
    ("dequant_without_127", "float c = (gamma * scale[m]) / 127.0f;", "float c = gamma * scale[m];"),
    ("bf16_truncates", "u += 0x7fffu + lsb;", "u += 0u * lsb;"),
    ("onebit_tie_to_plus", "codes[e] = (int8_t)(load_f(W, dt, e) > a ? 1 : -1);",
     "codes[e] = (int8_t)(load_f(W, dt, e) >= a ? 1 : -1);"),
    ("onebit_alpha_of_abs", "return fixed_order_sum(W, dt, N, K, 0);", "return fixed_order_sum(W, dt, N, K, 1);"),
    ("onebit_bits_reversed", "if (q > 0) byte |= 1u << i;", "if (q > 0) byte |= 0x80u >> i;"),
    ("backward_dx_without_gamma", "dx[m * K + k] = (float)((double)gamma * S);", "dx[m * K + k] = (float)S;"),
    ("backward_dx_sign", "load_f(dy, dydt, m * N + n), -1);", "load_f(dy, dydt, m * N + n), +1);"),
    ("exact_sum_drops_high_digit", "a->d[i + 1] += sign * hi;", "a->d[i + 1] += 0 * hi;"),
    ("exact_sum_without_sticky_bit", "if (round_bit && (sticky || (sig & 1u))) {", "if (round_bit && (sig & 1u)) {"),
    ("exact_sum_subnormal_shift", "int shift = e ? (int)e - 1 : 0;", "int shift = e ? (int)e : 0;"),
    ("backward_dw_without_scale", "T += t * c;", "T += t;"),
    ("backward_dw_k_reversed", "(double)xq[m * K + k];", "(double)xq[m * K + (K - 1 - k)];"),
    ("layernorm_unbiased_variance", "const double var = token_tree_sum(lane) / (double)K;",
     "const double var = token_tree_sum(lane) / (double)(K > 1 ? K - 1 : 1);"),
    ("layernorm_without_bias", "* (double)g[k] + (double)b[k];", "* (double)g[k];"),
    ("layernorm_without_eps", "sqrt(var + (double)eps)", "sqrt(var)"),
    ("layernorm_tree_drops_a_level", "for (int s = 128; s >= 1; s >>= 1)", "for (int s = 128; s >= 2; s >>= 1)"),
    ("ternarize_without_upper_clamp", "if (q > 1.0f) q = 1.0f;", ";"),
    ("ternarize_without_lower_clamp", "if (q < -1.0f) q = -1.0f;", ";"),
    ("ternarize_reciprocal_multiply", "float r = load_f(W, dt, e) / d;", "float r = load_f(W, dt, e) * (1.0f / d);"),
    ("pack_base3_first_weight_most_significant", "byte += digit * pow3;", "byte = byte * 3u + digit;"),
    ("pack_twos_complement_codes", "unsigned digit = (unsigned)(q + 1);", "unsigned digit = (unsigned)q & 3u;"),
    ("unpack_accepts_base3_bytes_above_242", "if (fmt == ORC_PACK_T5 && byte >= 243) return -1;", ";"),
    ("act_quant_signed_max", "float a = fabsf(load_f(x, dt, m * K + k));", "float a = load_f(x, dt, m * K + k);"),
    ("act_quant_reciprocal_multiply", "float t = load_f(x, dt, m * K + k) / s;",
     "float t = load_f(x, dt, m * K + k) * (1.0f / s);"),
    ("matmul_skips_minus_one", "s += (int32_t)codes[n * K + k] * (int32_t)xq[m * K + k];",
     "s += (codes[n * K + k] > 0) * (int32_t)xq[m * K + k];"),
    ("dequant_without_gamma", "float c = (gamma * scale[m]) / 127.0f;", "float c = scale[m] / 127.0f;"),
    ("dequant_reassociated", "float c = (gamma * scale[m]) / 127.0f;", "float c = gamma * (scale[m] / 127.0f);"),
    ("onebit_beta_of_signed", "sa += (double)fabsf(w[i]);", "sa += (double)w[i];"),
    ("backward_dx_skips_minus_one", "xsum_add(&acc, load_f(dy, dydt, m * N + n), -1);", ";"),
    ("layernorm_variance_about_zero", "const double d = (double)load_f(x, dt, m * K + k) - mu;",
     "const double d = (double)load_f(x, dt, m * K + k);"),
    ("layernorm_mean_over_lanes", "const double mu = token_tree_sum(lane) / (double)K;",
     "const double mu = token_tree_sum(lane) / 256.0;"),
    ("layernorm_without_sqrt", "const double r = 1.0 / sqrt(var + (double)eps);",
     "const double r = 1.0 / (var + (double)eps);"),
    ("unpack_accepts_nonzero_padding", "else if (digit != 1)", "else if (0)"),
    ("unpack_accepts_set_pad_bits", "else if (bit != 0)", "else if (0)"),
    ("onebit_matrix_compares_with_beta", "codes[e] = (int8_t)(load_f(W, dt, e) > a ? 1 : -1);",
     "codes[e] = (int8_t)(load_f(W, dt, e) > *beta ? 1 : -1);"),
]

GCC = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
       "-fno-strict-aliasing"]


def _build_planted(tmp, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"{name}: the text to replace must occur once"
    c_path = os.path.join(tmp, f"{name}.c")
    so_path = os.path.join(tmp, f"lib{name}.so")
    with open(c_path, "w") as f:
        f.write(src.replace(old, new))
    subprocess.run(GCC + ["-o", so_path, c_path, "-lm"], check=True)
    return so_path


def _pins_fail(so_path):
    env = dict(os.environ, BL_ORACLE_PLANTED_LIB=so_path, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                        *PIN_FILES], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode != 0, r.stdout[-2000:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    assert PIN_FILES and not any(p.endswith("test_pins_catch_mistakes.py") for p in PIN_FILES)
    libs = [(name, _build_planted(str(tmp_path), name, old, new)) for name, old, new in MISTAKES]
    with ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        results = list(ex.map(lambda nl: (nl[0], *_pins_fail(nl[1])), libs))
    missed = [name for name, failed, _ in results if not failed]
    assert not missed, f"no pin fails for: {missed}"


@pytest.mark.parametrize("name,old,new", MISTAKES[:1])
def test_unplanted_copy_passes(tmp_path, name, old, new):
    """Control: a copy built the same way without a mistake passes the pins."""
    so_path = _build_planted(str(tmp_path), "control", old, old)
    failed, out = _pins_fail(so_path)
    assert not failed, out
