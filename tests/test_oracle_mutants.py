"""The oracle's pins catch plausible mistakes.

Each case copies the oracle's C source to a temporary directory, plants one mistake (a
wrong bias, a dropped term, a transposed index, truncation instead of ties-to-even ...),
builds it there and runs the pin checks from the other oracle test modules against the
mutant.  At least one pin must fail for every mutant.  Nothing here touches a GPU.
"""
import importlib.util
import os
import subprocess

import numpy as np
import pytest

import test_oracle_codec as tc
import test_oracle_delayed as td
import test_oracle_mx as tmx
import test_oracle_mx_gemm as tmg
import test_oracle_health as th
import test_oracle_gemm as tg
import test_oracle_quantize as tq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fp8_oracle.c")

MUTANTS = {
    "e4m3_bias": ("f.bias = 7;", "f.bias = 8;"),
    "ties_away": ("if (rem > half || (rem == half && (r & 1))) r += 1;", "if (rem >= half) r += 1;"),
    "truncate": ("if (rem > half || (rem == half && (r & 1))) r += 1;", ""),
    "sat_to_nan": ("f.max_code = 0x7E;", "f.max_code = 0x7F;"),
    "flush_subnormal_enc": ("code = (int)r;                                       /* subnormal",
                            "code = 0;                                            /* subnormal"),
    "subnormal_dec_scale": ("ldexp((double)m, 1 - f.bias - f.mbits)", "ldexp((double)m, - f.bias - f.mbits)"),
    "scale_reciprocal": ("return amax / fm;", "return amax * (1.0f / fm);"),
    "quotient_reciprocal": ("float q = x / s;", "float q = x * (1.0f / s);"),
    "signed_amax": ("float v = fabsf(bf16_value(x[r * ld + c]));", "float v = bf16_value(x[r * ld + c]);"),
    "zero_group_divides": ("if (s == 0.0f) return (uint8_t)((f32_to_bits(x) >> 24) & 0x80u);", ""),
    "group_scale_layout": ("scales[g * rows + r] = quantize_region", "scales[r * cdiv(cols, 128) + g] = quantize_region"),
    "block_scale_transposed": ("return scales[(r / 128) * cdiv(cols, 128) + c / 128];",
                               "return scales[(c / 128) * cdiv(rows, 128) + r / 128];"),
    "kv_head_stride": ("quantize_region(fmt, x + h * D, T, D, ld, codes + h * D)",
                       "quantize_region(fmt, x + h * D, T, D, D, codes + h * D)"),
    "kv_tok_block_rows": ("int64_t t0 = tb * 128, nt = T - t0 < 128 ? T - t0 : 128;",
                          "int64_t t0 = tb * 128, nt = T - t0 < 64 ? T - t0 : 64;"),
    "bf16_truncate": ("if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1;", ""),
    "gemm_drop_sa": ("* (double)scale_at(sA, M, K, gA, rows[i], k);", ";"),
    "gemm_b_index": ("scale_at(sB, N, K, gB, n, k)", "scale_at(sB, N, K, gB, k % N, n % K)"),
    "gemm_b_transposed": ("b[k] = (double)orc_decode(fmtB, B[n * K + k])", "b[k] = (double)orc_decode(fmtB, B[(k % N) * K + (n % K)])"),
    "delayed_ignores_history": ("        if (step > 0) {\n            a = 0.0f;", "        if (0) {\n            a = 0.0f;"),
    "delayed_history_slot": ("history[(step % H) * ngroups + g] = cur[g];", "history[((step + 1) % H) * ngroups + g] = cur[g];"),
    "saturation_tie_flipped": ("return (f.max_code & 1) != 0;", "return (f.max_code & 1) == 0;"),
    "saturation_at_fmax": ("if (a > mid) return 1;", "if (a > (double)f.fmax) return 1;"),
    "underflow_counts_zeros": ("if (!isnan(xv) && xv != 0.0f && (code & 0x7F) == 0)", "if (!isnan(xv) && (code & 0x7F) == 0)"),
    "mx_exponent_not_minimal": ("(double)amax <= ldexp(fm, k - 1)) --k;", "(double)amax < ldexp(fm, k - 1)) --k;"),
    "mx_scale_bias": ("scales[r * (cols / 32) + g] = (uint8_t)(k + 127);", "scales[r * (cols / 32) + g] = (uint8_t)(k + 128);"),
    "mx_group_16": ("float amax = region_amax(xg, 1, 32, 32);", "float amax = region_amax(xg, 1, 16, 32);"),
    "mx_gemm_group_128": ("mx_scale_value(sA[rows[i] * G + k / 32])", "mx_scale_value(sA[rows[i] * G + k / 128])"),
    "mx_gemm_bias": ("ldexp(1.0, (int)b - 127)", "ldexp(1.0, (int)b - 126)"),
    "mx_gemm_b_scale_transposed": ("mx_scale_value(sB[n * G + k / 32])", "mx_scale_value(sB[(k / 32) * N + n])"),
    "mx_gemm_b_format_of_a": ("b[k] = (double)orc_decode(fmtB, B[n * K + k]) * mx_scale_value",
                              "b[k] = (double)orc_decode(fmtA, B[n * K + k]) * mx_scale_value"),
    "mx_gemm_nan_scale_ignored": ("return b == 255 ? NAN : ldexp", "return b == 255 ? 1.0 : ldexp"),
    "hist_bucket_shift": ("b = (int)((bits >> 23) & 0xFF);", "b = (int)((bits >> 24) & 0xFF);"),
    "hist_sign_in_bucket": ("b = (int)((bits >> 23) & 0xFF);", "b = (int)(((bits >> 23) + (bits >> 31)) & 0xFF);"),
    "underflow_counts_zero_inputs": ("if (!isnan(xv) && xv != 0.0f && (codes[i] & 0x7F) == 0) *count += 1;",
                                     "if (!isnan(xv) && (codes[i] & 0x7F) == 0) *count += 1;"),
    "mx_dequant_drops_scale": ("y[r * cols + c] = bf16_round(orc_decode(fmt, codes[r * cols + c]) * s);",
                               "y[r * cols + c] = bf16_round(orc_decode(fmt, codes[r * cols + c]));"),
}


def _pins(m):
    """Cheap pin checks, run against module `m` (the oracle or a mutant)."""
    checks = [
        lambda: tc.test_decode_matches_torch_float8(m, 0),
        lambda: tc.test_decode_matches_torch_float8(m, 1),
        lambda: tc.test_roundtrip_all_256_codes(m, 0),
        lambda: tc.test_roundtrip_all_256_codes(m, 1),
        lambda: tc.test_saturation(m, _gold(), 0, 0x7E),
        lambda: tc.test_ties_to_even_and_zero(m),
        lambda: tq.test_worked_example_fp8_vs_int8(m),
        lambda: tq.test_special_groups(m),
        lambda: tq.test_dequantize_matches_torch(m, 0, 2),
        lambda: tq.test_dequantize_matches_torch(m, 0, 1),
    ]
    for gran in (0, 1, 2):
        checks.append(lambda gran=gran: tq.test_quantize_bruteforce_tiny(m, 0, gran, (129, 257)))
    for gran in (0, 1, 2):
        checks.append(lambda gran=gran: tq.test_kv_bruteforce_tiny(m, 0, gran, (257, 8, 64)))
    checks += [
        lambda: td.test_hand_worked_e4m3_unit_scale(m),
        lambda: td.test_hand_worked_e5m2_unit_scale(m),
        lambda: td.test_ring_update_and_window_max(m),
        lambda: td.test_zero_history_gives_sign_only_codes(m),
        lambda: td.test_history_holding_the_current_amax_reduces_to_dynamic(m),
        lambda: tmx.test_exponent_at_powers_of_two_of_fmax(m, 0),
        lambda: tmx.test_bruteforce_tiny(m, 0, (3, 96)),
        lambda: tmx.test_dequantize_matches_torch(m, 0),
        lambda: th.test_histogram_hand_worked(m),
        lambda: th.test_histogram_matches_frexp(m),
        lambda: th.test_underflow_hand_worked(m),
        lambda: tmg.test_uniform_scales_reduce_to_matmul(m, 0, 1),
        lambda: tmg.test_one_group_special_case(m),
        lambda: tmg.test_row_and_column_doubling(m),
        lambda: tmg.test_nan_scale_poisons_its_row(m),
        lambda: tg.test_closed_form_constant_operands(m),
        lambda: tg.test_matches_numpy_matmul(m, 1, 2, (130, 384, 256)),
        lambda: tg.test_blockwise_identity(m),
    ]
    failed = 0
    for c in checks:
        try:
            c()
        except AssertionError:
            failed += 1
    return failed


def _gold():
    import json
    with open(tc.GOLD) as f:
        return json.load(f)


def _mutant_module(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, old
    path = tmp_path / "fp8_oracle.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           "-fno-fast-math", "-o", str(lib), str(path), "-lm"])
    spec = importlib.util.spec_from_file_location("oracle_mutant", os.path.join(ROOT, "oracle", "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC, mod._LIB, mod._lib = str(path), str(lib), None
    return mod


def test_pins_pass_on_the_oracle(orc):
    assert _pins(orc) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    with np.errstate(all="ignore"):
        assert _pins(_mutant_module(tmp_path, old, new)) > 0, f"mutant {name} survived every pin"
