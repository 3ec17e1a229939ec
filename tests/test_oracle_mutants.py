"""The pins have teeth: each plausible mistake planted in a copy of the oracle
(on the CPU, in a temporary directory) must make tests/test_oracle_pins.py fail."""
import os
import subprocess
import sys
import tempfile

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "round_half_away": ("rintf(x[i] / s)", "roundf(x[i] / s)"),
    "nibble_order_swapped": ("out[i] = (uint8_t)(lo | (hi << 4));",
                             "out[i] = (uint8_t)(hi | (lo << 4));"),
    "scale_not_rounded_to_bf16": ("float s = oracle_bf16_to_f32(s_bits);", "float s = s32;"),
    "range_not_widened_to_zero": ("float mn = 0.0f, mx = 0.0f;", "float mn = x[0], mx = x[0];"),
    "sixteen_levels": ("(mx - mn) / 15.0f", "(mx - mn) / 16.0f"),
    "sym_divides_by_8": ("amax / 7.0f", "amax / 8.0f"),
    "zero_point_sign": ("rintf(-mn / s)", "rintf(mn / s)"),
    "gemm_weight_transposed": ("(double)oracle_bf16_to_f32(W_hat[n * K + k]);",
                               "(double)oracle_bf16_to_f32(W_hat[k * N + n]);"),
    "dequant_truncates": ("return oracle_f32_to_bf16_rn(prod);",
                          "uint32_t u; memcpy(&u, &prod, 4); return (uint16_t)(u >> 16);"),
    "group_index_wraps": ("int64_t j = k / g;", "int64_t j = k % G;"),
    # 8-bit (W8A16) functions
    "w8_256_levels": ("(mx - mn) / 255.0f", "(mx - mn) / 256.0f"),
    "w8_sym_divides_by_128": ("amax / 127.0f", "amax / 128.0f"),
    "w8_int8_sign_extension": ("if (sym && q >= 128) q -= 256;", "if (sym && q >= 128) q -= 128;"),
    "w8_code_bytes_reversed": ("codes[n * K + j * g + i] = (uint8_t)",
                               "codes[n * K + j * g + (g - 1 - i)] = (uint8_t)"),
    "w8_zero_point_clamped_to_15": ("rintf(-mn / s), 0.0f, 255.0f", "rintf(-mn / s), 0.0f, 15.0f"),
    "w8_dequant_truncates": ("W_hat[n * K + k] = oracle_f32_to_bf16_rn(prod);",
                             "uint32_t u; memcpy(&u, &prod, 4); W_hat[n * K + k] = (uint16_t)(u >> 16);"),
    # per-K activation scale
    "act_scale_truncates": ("Xs[m * K + k] = oracle_f32_to_bf16_rn(prod);",
                            "uint32_t u; memcpy(&u, &prod, 4); Xs[m * K + k] = (uint16_t)(u >> 16);"),
    "act_scale_indexed_by_row": ("oracle_bf16_to_f32(a[k]);", "oracle_bf16_to_f32(a[m % K]);"),
    # W8A8 (per-token INT8 activations x per-channel INT8 weights)
    "w8a8_act_divides_by_128": ("float sc = amax / 127.0f;", "float sc = amax / 128.0f;"),
    "w8a8_act_truncates": ("float r = rintf(oracle_bf16_to_f32(X[m * K + k]) / sc);",
                           "float r = truncf(oracle_bf16_to_f32(X[m * K + k]) / sc);"),
    "w8a8_scale_of_first_token": ("float a = fabsf(oracle_bf16_to_f32(X[m * K + k]));",
                                  "float a = fabsf(oracle_bf16_to_f32(X[k]));"),
    "w8a8_gemm_drops_weight_scale": ("(double)sx[m] * (double)oracle_bf16_to_f32(sw[n]) * (double)acc;",
                                     "(double)sx[m] * (double)acc;"),
    "w8a8_gemm_weight_transposed": ("(int64_t)qw[n * K + k];\n            Y[m * N + n]",
                                    "(int64_t)qw[(k * N + n) % (N * K)];\n            Y[m * N + n]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert old in text, f"mutation anchor for {name} not found"
    src = tmp_path / "oracle_mutant.c"
    src.write_text(text.replace(old, new))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(lib), str(src), "-lm"])
    env = dict(os.environ, W4A16_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
