"""The oracle pins must catch plausible mistakes.

Each case compiles a copy of the oracle's C source with one deliberate slip (a wrong
rounding mode, an off-by-one exponent, a swapped nibble, a transposed operand, ...)
and runs the pin tests against it in a subprocess; the pins must fail.  The mistake
is planted only in a temporary CPU-side copy of the oracle.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "mx_oracle.c")

MUTANTS = [
    ("ties_away_from_zero", "double n = nearbyint(a / q);", "double n = round(a / q);"),
    ("scale_exponent_off_by_one", "int sc = (e2 - 1) + 127 - f->emax;", "int sc = e2 + 127 - f->emax;"),
    ("e4m3_emax_7", "{4, 3, 7, 8, 448.0}", "{4, 3, 7, 7, 448.0}"),
    ("no_saturation", [("if (v > f->maxval) v = f->maxval;       /* rounding",
                        "if (0) v = f->maxval;       /* rounding"),
                       ("if (a >= f->maxval) {", "if (a >= 4 * f->maxval) {")]),
    ("negative_zero_dropped", "int sign = signbit(y) ? 1 : 0;", "int sign = (y < 0) ? 1 : 0;"),
    ("nibbles_swapped", "} else if ((k & 1) == 0) {", "} else if ((k & 1) == 1) {"),
    ("no_subnormal_floor", "if (e < emin) e = emin;                 /* subnormal",
     "if (0) e = emin;                 /* subnormal"),
    ("scale_multiplied", "else codes[i] = mxo_encode_elem(v[i] / mxo_scale_value(sc), fmt);",
     "else codes[i] = mxo_encode_elem(v[i] * mxo_scale_value(sc), fmt);"),
    ("weights_transposed", "const double *w = j->wdeq + n * K;", "const double *w = j->wdeq + n;"),
    ("bias_dropped", "if (j->bias) acc += mxo_bf16_to_double(j->bias[n]);", "(void)0;"),
    ("sf_atom_rows_swapped", "return atom * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (kb % 4);",
     "return atom * 512 + (r % 32) * 4 + ((r / 32) % 4) * 16 + (kb % 4);"),
    ("dequant_wrong_block_index", "mxo_scale_value(sf[r * KB + k / 32]);",
     "mxo_scale_value(sf[r * KB + (k / 32 + 1) % KB]);"),
    ("bf16_round_truncates", "double r = nearbyint(a / q) * q;", "double r = floor(a / q) * q;"),
    ("bf16_ties_away_from_zero", "double r = nearbyint(a / q) * q;", "double r = round(a / q) * q;"),
    ("bf16_overflow_saturates", "if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);",
     "if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F7Fu);"),
    ("gelu_without_sqrt2", "erfc(-x / sqrt(2.0));", "erfc(-x);"),
    ("gelu_tanh_form", "double mxo_gelu(double x) { return 0.5 * x * erfc(-x / sqrt(2.0)); }",
     "double mxo_gelu(double x) { return 0.5 * x * (1.0 + tanh(sqrt(2.0 / M_PI) * (x + 0.044715 * x * x * x))); }"),
    ("static_scale_dropped", "y[i * N + j] = alpha * y[i * N + j] + (bias",
     "y[i * N + j] = y[i * N + j] + (bias"),
    ("static_bias_scaled", "y[i * N + j] = alpha * y[i * N + j] + (bias ? mxo_bf16_to_double(bias[j]) : 0.0);",
     "y[i * N + j] = alpha * (y[i * N + j] + (bias ? mxo_bf16_to_double(bias[j]) : 0.0));"),
    ("static_binary32_quotient", "double q = mxo_bf16_to_double(x[i]) / (double)scale;",
     "double q = (float)(mxo_bf16_to_double(x[i]) / (double)scale);"),
    ("static_binary32_product", "double q = mxo_bf16_to_double(x[i]) / (double)scale;",
     "double q = (float)(mxo_bf16_to_double(x[i]) * (double)(float)(1.0 / scale));"),
    ("static_scale_multiplies", "double q = mxo_bf16_to_double(x[i]) / (double)scale;",
     "double q = mxo_bf16_to_double(x[i]) * (double)scale;"),
    ("hadamard_sign_rule", "double h = (__builtin_popcount((unsigned)(j & k)) & 1) ? -1.0 : 1.0;",
     "double h = (__builtin_popcount((unsigned)(j | k)) & 1) ? -1.0 : 1.0;"),
    ("hadamard_unnormalized", "const double inv_sqrt_b = 1.0 / sqrt((double)B);", "const double inv_sqrt_b = 1.0;"),
    ("smoothing_divides", "a[k] = mul ? xk * (double)mul[k] : xk;", "a[k] = mul ? xk / (double)mul[k] : xk;"),
    ("transform_bound_dropped",
     "delta[b0 + j] = 1.01 * ((d + 4) * u * s1 + (B + 2) * ldexp(1.0, -150)) * inv_sqrt_b;",
     "delta[b0 + j] = 0.0;"),
    ("transform_scale_flag_dropped", "if (!amb && mxo_scale_code(lo, 0, fmt) != mxo_scale_code(hi, 0, fmt)) amb = 1;",
     "(void)0;"),
    ("transform_overflow_unflagged", "if (l1[kb * 32 + i] >= ldexp(1.0, 127)) amb = 2;", "(void)0;"),
    ("lowrank_u_not_rounded", "            u[j] = mxo_bf16_to_double(mxo_double_to_bf16(acc));", "            u[j] = acc;"),
    ("lowrank_l2_transposed", "for (int64_t j = 0; j < r; ++j) acc += u[j] * mxo_bf16_to_double(l2t[n * r + j]);",
     "for (int64_t j = 0; j < r; ++j) acc += u[j] * mxo_bf16_to_double(l2t[(j * N + n) % (N * r)]);"),
    ("gelu_cancelling_form", "double mxo_gelu(double x) { return 0.5 * x * erfc(-x / sqrt(2.0)); }",
     "double mxo_gelu(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }"),
]


def _edits(m):
    return m[1] if isinstance(m[1], list) else [(m[1], m[2])]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(mutant, tmp_path):
    name = mutant[0]
    src = open(SRC).read()
    for old, new in _edits(mutant):
        assert src.count(old) == 1, "mutation anchor not found: " + name
        src = src.replace(old, new)
    mut = tmp_path / ("mx_oracle_%s.c" % name)
    mut.write_text(src)
    so = tmp_path / ("libmx_oracle_%s.so" % name)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-D_GNU_SOURCE",
                           str(mut), "-o", str(so), "-lm", "-lpthread"])
    env = dict(os.environ, MXO_LIB_OVERRIDE=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "pins did not catch mutant %s:\n%s" % (name, r.stdout[-2000:])
