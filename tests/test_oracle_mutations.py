"""The pins catch plausible mistakes: each case plants one slip in a copy of
the oracle's source (on the CPU, in a temporary directory), builds it, and
checks that the named pin test fails against that build."""
from __future__ import annotations

import concurrent.futures
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = [
    ("s * (1.0 + g * (1.0 - s))", "s * (1.0 + g * (1.0 + s))", "test_silu_grad_matches_finite_difference"),
    ("s * (1.0 + g * (1.0 - s))", "s * (1.0 + (1.0 - s))", "test_silu_grad_matches_finite_difference"),
    ("*d_gate = dy * u * oracle_silu_grad(g);", "*d_gate = dy * oracle_silu_grad(g);", "test_swiglu_bwd_fp64_finite_differences"),
    ("*d_up = dy * silu;", "*d_up = dy * u;", "test_swiglu_bwd_fp64_matches_torch_autograd"),
    ("x[m * 2 * K + k]);", "x[m * 2 * K + K + k]);", "test_whole_op_gate32_closed_form"),
    ("const float qmax = codes ? 448.0f : 127.0f;", "const float qmax = codes ? 448.0f : 128.0f;",
     "test_quant_scale_is_amax_over_127_rounded_once"),
    ("float r = std::nearbyint(t);", "float r = std::round(t);", "test_quant_ties_to_even_and_symmetry"),
    ("(j < Kg) ? &dg[m * K + j * G] : &du[m * K + (j - Kg) * G]",
     "(j < Kg) ? &du[m * K + j * G] : &dg[m * K + (j - Kg) * G]", "test_whole_op_gate32_closed_form"),
    ("&y_q_t[k * M + t0], 1,", "&y_q_t[t0 * K + k], K,", "test_whole_op_gate32_closed_form"),
    ("const int64_t si = ys_layout ? (i * K + k) : (k * Mg + i);",
     "const int64_t si = ys_layout ? (i * K + k) : (i * K + k);", "test_whole_op_gate32_closed_form"),
    ("gis + (m * 2 * Kg + j) * sb", "gis + (j * M + m) * sb", "test_whole_op_groups_relate_to_stage1"),
    ("const double r = std::nearbyint(a / ulp) * ulp;", "const double r = std::trunc(a / ulp) * ulp;",
     "test_bf16_rne_bruteforce_exact_rationals"),
    ("    s = 1.0;\n", "    s = 2.0;\n", "test_quant_zero_and_constant_groups"),
    ("if (e < -126) e = -126;", "", "test_bf16_rne_against_torch_float32_conversion"),
    ("return 1.0 / (1.0 + std::exp(-g));", "return 1.0 / (1.0 + std::exp(-(float)g));",
     "test_sigmoid_matches_library_expit"),
    # output formats (pins in test_oracle_formats.py)
    ("if (e < -6) e = -6;", "", "test_e4m3_rne_bruteforce_exact_rationals", "formats"),
    ("std::ldexp(1.0, e - 3)", "std::ldexp(1.0, e - 4)", "test_e4m3_rne_against_torch_float8_conversion",
     "formats"),
    ("const double r = std::nearbyint(a / ulp) * ulp;  // a/ulp is exact; nearbyint ties to even\n"
     "  if (r < std::ldexp(1.0, -6))",
     "const double r = std::round(a / ulp) * ulp;\n  if (r < std::ldexp(1.0, -6))",
     "test_e4m3_rne_bruteforce_exact_rationals", "formats"),
    ("if (a > 448.0) return sign | 0x7E;", "if (a > 480.0) return sign | 0x7E;",
     "test_e4m3_rne_bruteforce_exact_rationals", "formats"),
    ("if (std::ldexp(1.0, k) < d) k += 1;", "", "test_e8m0_ceil_bruteforce", "formats"),
    ("if (k < -127) k = -127;", "", "test_e8m0_ceil_bruteforce", "formats"),
    ("const float qmax = codes ? 448.0f : 127.0f;", "const float qmax = codes ? 447.0f : 127.0f;",
     "test_quant_group_fmt_bruteforce", "formats"),
    ("s = scales ? oracle_e8m0_value(oracle_e8m0_ceil(s32)) : static_cast<double>(s32);",
     "s = static_cast<double>(s32);", "test_quant_group_fmt_bruteforce", "formats"),
    ("const int64_t si = ys_layout ? (i * K + k) : (k * Mg + i);",
     "const int64_t si = ys_layout ? (k * Mg + i) : (k * Mg + i);",
     "test_whole_op_fmt_ys_layouts_transpose", "formats"),
    ("oracle_quant_group_fmt(&y[t0 * K + k], n, K,", "oracle_quant_group_fmt(&y[t0 * K + k], n, 1,",
     "test_whole_op_fmt_groups_relate_to_stage1", "formats"),
    # forward-side neighbour (pins in test_oracle_fwd.py)
    ("if (e < -14) e = -14;", "", "test_fp16_rne_against_numpy_float16_conversion", "fwd"),
    ("const int mant = static_cast<int>(r / std::ldexp(1.0, re - 10)) - 1024;",
     "const int mant = static_cast<int>(r / std::ldexp(1.0, re - 10)) - 1023;",
     "test_fp16_rne_against_numpy_float16_conversion", "fwd"),
    ("gv = gv < limit ? gv : limit;", "gv = gv < -limit ? -limit : (gv > limit ? limit : gv);",
     "test_swiglu_rows_limit_clamps_gate_above_and_up_both_ways", "fwd"),
    ("h[k] = oracle_bf16_rne(oracle_silu(gv) * uv * w);", "h[k] = oracle_bf16_rne(oracle_silu(gv) * uv);",
     "test_swiglu_rows_closed_form_without_clamp", "fwd"),
    ("s16 = oracle_fp16_rne(static_cast<double>(d) * static_cast<double>(qsum));  // exact product",
     "s16 = oracle_fp16_rne(static_cast<double>(qsum));", "test_q8_1_block_against_its_definition", "fwd"),
    ("&q8[(m * (inter / 32) + b) * 36]", "&q8[(b * rows + m) * 36]",
     "test_swiglu_rows_blocks_are_the_rows_32_value_blocks", "fwd"),
    ("if (limit > 0.0) {   // false for NaN: no clamp", "if (limit != 0.0) {",
     "test_swiglu_rows_closed_form_without_clamp", "fwd"),
    # the whole op against its brute-force restatement (test_oracle_bruteforce.py)
    ("*d_up = dy * silu;", "*d_up = dy * silu * u;", "test_whole_oracle_equals_bruteforce_on_4x128", "brute"),
    ("x[m * 2 * K + k]);", "x[m * 2 * K + K + k]);", "test_whole_oracle_equals_bruteforce_on_4x128", "brute"),
    ("const float qmax = codes ? 448.0f : 127.0f;", "const float qmax = codes ? 448.0f : 127.5f;",
     "test_whole_oracle_equals_bruteforce_on_4x128", "brute"),
    # groups of G channels when G does not divide K (pins in test_oracle_formats.py)
    ("const int64_t n = (K - c0 < G) ? K - c0 : G;", "const int64_t n = G < K ? G : K;",
     "test_short_last_group_equals_the_zero_padded_op", "formats"),
    ("&grad_input_q[m * 2 * K + (j < Kg ? 0 : K) + c0]", "&grad_input_q[m * 2 * K + j * G]",
     "test_short_last_group_equals_the_zero_padded_op", "formats"),
    # a quantized grad_y (pins in test_oracle_qgrad.py)
    ("static_cast<double>(s[m * Kg + k / 128])", "static_cast<double>(s[m * Kg + k % Kg])",
     "test_whole_op_pow2_scales_equals_bf16_op", "qgrad"),
    ("static_cast<double>(s[m * Kg + k / 128])", "static_cast<double>(s[(k / 128) * M + m])",
     "test_whole_op_pow2_scales_equals_bf16_op", "qgrad"),
    ("static_cast<double>(q[m * K + k])", "static_cast<double>(static_cast<uint8_t>(q[m * K + k]))",
     "test_first_stage_against_autograd", "qgrad"),
    ("static_cast<double>(q[m * K + k]) * static_cast<double>(s[m * Kg + k / 128])",
     "static_cast<double>(static_cast<float>(q[m * K + k]) * s[m * Kg + k / 128])",
     "test_dequant_is_exact_in_fp64", "qgrad"),
]

PIN_FILES = {"pins": "test_oracle_pins.py", "formats": "test_oracle_formats.py",
             "fwd": "test_oracle_fwd.py", "qgrad": "test_oracle_qgrad.py",
             "brute": "test_oracle_bruteforce.py"}


def _run_mutant(tmp_dir, idx, old, new, pin, pins="pins"):
    src = open(oracle._SRC).read()
    if src.count(old) < 1:
        return f"mutation #{idx} no longer applies: {old!r}"
    mutated = os.path.join(tmp_dir, f"mut{idx}.cpp")
    with open(mutated, "w") as f:
        f.write(src.replace(old, new, 1))
    so = os.path.join(tmp_dir, f"libmut{idx}.so")
    subprocess.run(["g++", *oracle.CXXFLAGS, mutated, "-o", so], check=True)
    env = dict(os.environ, SDQ_ORACLE_LIB=so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", PIN_FILES[pins]), "-k", pin],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    if r.returncode == 0:
        return f"planted mistake #{idx} survived {pin}: {old!r} -> {new!r}"
    return None


def test_pins_catch_planted_mistakes(tmp_path):
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(2, os.cpu_count() or 2)) as ex:
        futs = [ex.submit(_run_mutant, str(tmp_path), i, *m) for i, m in enumerate(MUTATIONS)]
        problems = [f.result() for f in futs]
    problems = [p for p in problems if p]
    assert not problems, "\n".join(problems)
