"""The CPU oracle against its pins (hand cases, closed forms, invariants, independent
library routines), and a check that those pins catch plausible mistakes planted in a
copy of the oracle source."""
import os
import subprocess

import pytest

import oracle
from oracle import build as obuild
import oracle_pins

pytestmark = pytest.mark.cpu


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


# Each mutant is one plausible slip in the oracle: (name, text in the source, replacement).
MUTANTS = [
    ("round_half_away", "float q = rintf(W[i] / gamma);", "float q = roundf(W[i] / gamma);"),
    ("reciprocal_multiply", "float q = rintf(W[i] / gamma);",
     "float q = rintf(W[i] * (1.0f / gamma));"),
    ("no_abs_in_gamma", "sum += fabs((double)W[n * K + k]);", "sum += (double)W[n * K + k];"),
    ("eps_dropped", "float gamma = mean + eps;", "float gamma = mean;"),
    ("mean_over_K_only", "float mean = (float)(sum / (double)(N * K));",
     "float mean = (float)(sum / (double)K);"),
    ("clip_to_two", "if (q > 1.0f) q = 1.0f;", "if (q > 2.0f) q = 2.0f;"),
    ("codes_swapped", "if (c == 1) return 1;\n    if (c == -1) return 2;",
     "if (c == 1) return 2;\n    if (c == -1) return 1;"),
    ("msb_first", "byte |= (unsigned)e << (2 * i);", "byte |= (unsigned)e << (6 - 2 * i);"),
    ("qb_128", "\n        float s = 127.0f / fmaxf(a, eps);", "\n        float s = 128.0f / fmaxf(a, eps);"),
    ("act_round_away", "float q = rintf(bf16_bits_to_float(X[m * K + k]) * s);",
     "float q = roundf(bf16_bits_to_float(X[m * K + k]) * s);"),
    ("act_no_abs", "float v = fabsf(bf16_bits_to_float(X[m * K + k]));",
     "float v = bf16_bits_to_float(X[m * K + k]);"),
    ("transposed_codes", "int8_t c = codes[n * K + k];", "int8_t c = codes[k * N + n];"),
    ("minus_is_plus", "else if (c == -1) sum -= xq[m * K + k];", "else if (c == -1) sum += xq[m * K + k];"),
    ("scale_inverted", "(double)acc[m * N + n] * (double)gamma / (double)s[m]",
     "(double)acc[m * N + n] * (double)gamma * (double)s[m]"),
    ("gamma_dropped", "(double)acc[m * N + n] * (double)gamma / (double)s[m]",
     "(double)acc[m * N + n] / (double)s[m]"),
    ("bf16_truncate", "u += 0x7FFFu + lsb;", "u += 0u * lsb;"),
    ("unpack_wrong_shift", "unsigned c = (byte >> (2 * (k % 4))) & 3u;",
     "unsigned c = (byte >> (2 * (3 - k % 4))) & 3u;"),
    ("layernorm_no_mean", "mu = mu / (double)K;", "mu = 0.0;"),
    ("norm_variance_unbiased", "v = v / (double)K;", "v = v / (double)(K - 1);"),
    ("norm_weight_ignored", "const float wk = (w != NULL) ? w[k] : 1.0f;", "const float wk = 1.0f;"),
    ("norm_eps_dropped", "const float r32 = (float)(1.0 / sqrt(v + (double)norm_eps));",
     "const float r32 = (float)(1.0 / sqrt(v));"),
    ("norm_round_away", "float q = rintf(xn[k] * s);", "float q = roundf(xn[k] * s);"),
    ("norm_elementwise_fp64", "const float t32 = d32 * r32;\n            xn[k] = t32 * wk;",
     "(void)d32;\n            xn[k] = (float)(((double)bf16_bits_to_float(X[m * K + k]) - mu) * "
     "(1.0 / sqrt(v + (double)norm_eps)) * (double)wk);"),
    ("norm_qb_128", "const float s = 127.0f / fmaxf(a, eps);", "const float s = 128.0f / fmaxf(a, eps);"),
    ("row_gamma_by_token", "(double)gamma_rows[n] / (double)s[m]", "(double)gamma_rows[m] / (double)s[m]"),
    ("row_gamma_dropped", "(double)acc[m * N + n] * (double)gamma_rows[n] / (double)s[m]",
     "(double)acc[m * N + n] / (double)s[m]"),
    ("tl5_floor_encode", "(uint8_t)((v * 256u + 242u) / 243u)", "(uint8_t)((v * 256u) / 243u)"),
    ("tl5_digit_order", "for (i = 0; i < 4 - p; ++i) w *= 3u;", "for (i = 0; i < p; ++i) w *= 3u;"),
    ("tl5_no_offset", "t = code + 1;", "t = code < 0 ? 2 : code;"),
    ("tl5_interleaved", "int64_t k = 80 * b + 16 * p + j;", "int64_t k = 80 * b + 5 * j + p;"),
    ("tl5_pad_minus_one", "int t = 1;\n", "int t = 0;\n"),
    ("tl5_decode_255", "unsigned v = byte * 243u / 256u;", "unsigned v = byte * 243u / 255u;"),
    ("ste_dx_no_gamma", "dX[m * K + k] = (float)((double)gamma * sum);", "dX[m * K + k] = (float)sum;"),
    ("ste_dx_codes_transposed", "sum += (double)dY[m * N + n] * (double)codes_tmp[n * K + k];",
     "sum += (double)dY[m * N + n] * (double)codes_tmp[k * N + n];"),
    ("ste_dw_times_s", "sum += (double)dY[m * N + n] * (double)xq[m * K + k] / (double)s[m];",
     "sum += (double)dY[m * N + n] * (double)xq[m * K + k] * (double)s[m];"),
    ("ste_dw_no_gamma", "dW[n * K + k] = (float)((double)gamma * sum);", "dW[n * K + k] = (float)sum;"),
    ("ste_dw_token_index", "sum += (double)dY[m * N + n] * (double)xq[m * K + k] / (double)s[m];",
     "sum += (double)dY[m * N + n] * (double)xq[m * K + k] / (double)s[0];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_oracle_mutant_is_caught(tmp_path, name, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, "mutation anchor not found: %s" % name
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / ("lib_%s.so" % name)
    subprocess.run(["gcc", *obuild.CFLAGS, str(mutated), "-o", str(lib), "-lm"], check=True,
                   stderr=subprocess.DEVNULL)
    M = oracle.Oracle(str(lib))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(M)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, "no pin caught mutant %s" % name
