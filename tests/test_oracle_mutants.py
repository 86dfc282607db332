"""Mutation check of the oracle pins.

Each entry plants one plausible mistake in a copy of the oracle's C source,
builds it, and runs the oracle pin tests against that build (through the
QZ_ORACLE_LIB override).  Every mutant must make at least one pin fail: a
surviving mutant would mean a part of the oracle that nothing but itself
vouches for.  Mistakes are planted only in the oracle, on the CPU.
"""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["tests/test_oracle_formats.py", "tests/test_oracle_mxfp8.py", "tests/test_oracle_layout.py",
             "tests/test_oracle_nvfp4.py", "tests/test_oracle_norm.py", "tests/test_oracle_dequant.py",
             "tests/test_oracle_merge.py", "tests/test_oracle_split.py", "tests/test_oracle_allreduce.py"]

MUTANTS = {
    "ties_away_from_even": ("return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "return f + 1.0;"),
    "ties_toward_zero": ("return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "return f;"),
    "e4m3_no_saturation": ("if (a > 448.0) a = 448.0;                /* saturate */", ""),
    "e8m0_floor_rule": ("while (amax > ldexp(448.0, e)) e += 1;", "e = E - 1 - 8;"),
    "e8m0_off_by_one": ("while (amax > ldexp(448.0, e)) e += 1;", "while (amax >= ldexp(448.0, e)) e += 1;"),
    "e8m0_no_clamp": ("    if (e < -127) e = -127;\n    return e;", "    return e;"),
    "mx_rcp_no_ftz": ("if (r < ldexp(1.0, -126)) return 0.0f;", ""),
    "nvfp4_no_zero_guard": ("if ((s & 0x7F) != 0) {", "if (1) {"),
    "nvfp4_scale_448": ("float g = A / 2688.0f;", "float g = A / 448.0f;"),
    "nvfp4_block_no_div6": ("float v = (b / 6.0f) * S;", "float v = b * S;"),
    "nvfp4_scale_direct": ("    float g = A / 2688.0f;            /* stored decode scale, 2688 = 448 * 6 */\n"
                           "    if (g == 0.0f) return 0.0f;\n    return 1.0f / g;",
                           "    float g = A / 2688.0f;            /* stored decode scale, 2688 = 448 * 6 */\n"
                           "    if (g == 0.0f) return 0.0f;\n    return 2688.0f / A;"),
    "nvfp4_block_fused_product": ("float v = (b / 6.0f) * S;", "float v = (b * S) / 6.0f;"),
    "nvfp4_rcp_as_product": ("rcp = S / (float)qzo_e4m3_value(s);", "rcp = S * (1.0f / (float)qzo_e4m3_value(s));"),
    "nibbles_swapped": ("(uint8_t)(qzo_e2m1_encode(y0) | (qzo_e2m1_encode(y1) << 4))",
                        "(uint8_t)((qzo_e2m1_encode(y0) << 4) | qzo_e2m1_encode(y1))"),
    "swizzle_plain_rowmajor": ("int64_t inner = ((r % 32) * 4 + (r / 32)) * 4 + (k % 4);",
                               "int64_t inner = r * 4 + (k % 4);"),
    "swizzle_floor_col_tiles": ("int64_t col_tiles = (kv + 3) / 4;", "int64_t col_tiles = kv / 4;"),
    "sf_padding_not_cleared": ("for (int64_t i = 0; i < n; i++) sf[i] = 0;", ""),
    "rms_sum_not_mean": ("double rstd = 1.0 / sqrt(ss / (double)H + (double)eps);",
                         "double rstd = 1.0 / sqrt(ss + (double)eps);"),
    "rms_eps_outside_sqrt": ("double rstd = 1.0 / sqrt(ss / (double)H + (double)eps);",
                             "double rstd = 1.0 / (sqrt(ss / (double)H) + (double)eps);"),
    "rms_gamma_row_index": ("gamma[i]);", "gamma[t]);"),
    "rms_square_unrounded_sum": ("ss += hv * hv;", "ss += s * s;"),
    "mx_row_stride_ignored": ("const uint16_t *blk = x + r * ld + k * 32;", "const uint16_t *blk = x + r * cols + k * 32;"),
    "dq_nibbles_swapped": ("uint8_t code = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);",
                           "uint8_t code = (c & 1) ? (uint8_t)(byte & 0xF) : (uint8_t)(byte >> 4);"),
    "dq_no_decode_scale": ("double v = qzo_e2m1_value(code) * qzo_e4m3_value(s) * (double)g;",
                           "double v = qzo_e2m1_value(code) * qzo_e4m3_value(s);"),
    "dq_binary32_product": ("double v = qzo_e2m1_value(code) * qzo_e4m3_value(s) * (double)g;",
                            "double v = (double)(float)(qzo_e2m1_value(code) * qzo_e4m3_value(s) * (double)g);"),
    "dq_mx_exponent_off_by_one": ("double v = qzo_e4m3_value(q[r * cols + c]) * ldexp(1.0, byte - 127);",
                                  "double v = qzo_e4m3_value(q[r * cols + c]) * ldexp(1.0, byte - 126);"),
    "dq_mx_linear_sf_index": ("int byte = sf[sf_offset(layout, r, c / 32, kv)];", "int byte = sf[r * kv + c / 32];"),
    "merge_no_normalisation": ("y[t * H + i] = qzo_bf16_from_double(acc / wsum);",
                               "y[t * H + i] = qzo_bf16_from_double(acc);"),
    "merge_no_max_shift": ("wsum += exp((double)lse[s * T + t] - m);", "wsum += exp((double)lse[s * T + t]);"),
    "merge_split_token_index": ("(double)O[(s * T + t) * H + i];", "(double)O[(t * S + s) * H + i];"),
    "split_no_block_check": ("    if (cut % row_block != 0 && cut < rows) return -1;\n", ""),
    "split_proportional_rule": ("    if (cut % row_block != 0 && cut < rows) return -1;\n",
                                "    if (rows > 0 && (((rows + row_block - 1) / row_block) * cut) % rows != 0) return -1;\n"),
    "split_second_part_offset": ("int64_t first[2] = {0, cut};", "int64_t first[2] = {0, cut - 1};"),
    "split_padding_not_cleared": ("            sf_clear(so[p], count[p], kv, dst_layout);\n", ""),
    "split_source_layout_ignored": ("= sf[sf_offset(src_layout, first[p] + r, k, kv)];",
                                    "= sf[sf_offset(dst_layout, first[p] + r, k, kv)];"),
    "split_amax_not_shared": ("if (amax_kind == 1) ao[p][0] = amax[0];",
                              "if (amax_kind == 1 && p == 0) ao[p][0] = amax[0];"),
    "split_block_scale_rows_floor": ("int64_t srows = (count[p] + 127) / 128;", "int64_t srows = count[p] / 128;"),
    "rank_sum_binary64": ("float acc = qzo_bf16_value(xs[0][i]);", "double acc = qzo_bf16_value(xs[0][i]);"),
    "rank_sum_drops_last_rank": ("for (int r = 1; r < n; r++) acc", "for (int r = 1; r < n - 1; r++) acc"),
    "rank_sum_reverse_order": ("float acc = qzo_bf16_value(xs[0][i]);\n        for (int r = 1; r < n; r++) acc",
                               "float acc = qzo_bf16_value(xs[n - 1][i]);\n        for (int r = n - 2; r >= 0; r--) acc"),
    "rank_sum_first_rank_only": ("out[i] = qzo_bf16_from_double((double)acc);",
                                 "out[i] = xs[0][i];"),
    "bf16_double_rounding": ("double n = round_half_even(a / step);\n    double r = n * step;",
                             "double n = round_half_even((double)(float)a / step);\n    double r = n * step;"),
}


def _build_mutant(name, old, new, tmp):
    src = open(os.path.join(ROOT, "oracle", "qz_oracle.c")).read()
    assert src.count(old) >= 1, f"mutant {name}: pattern not found"
    path_c = os.path.join(tmp, f"{name}.c")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    return oracle.compile_library(path_c, os.path.join(tmp, f"{name}.so"))


def _run_pins(lib_path):
    env = dict(os.environ, QZ_ORACLE_LIB=lib_path)
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PIN_FILES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return p.returncode


def test_every_mutant_fails_a_pin():
    tmp = tempfile.mkdtemp(prefix="qz_mutants_")
    try:
        libs = {n: _build_mutant(n, o, w, tmp) for n, (o, w) in MUTANTS.items()}
        with ThreadPoolExecutor(max_workers=max(1, min(8, oracle.host_threads()))) as ex:
            codes = dict(zip(libs, ex.map(_run_pins, libs.values())))
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    survivors = [n for n, rc in codes.items() if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"


def test_unmutated_build_passes_pins():
    tmp = tempfile.mkdtemp(prefix="qz_mutants_")
    try:
        lib = oracle.compile_library(os.path.join(ROOT, "oracle", "qz_oracle.c"), os.path.join(tmp, "clean.so"))
        assert _run_pins(lib) == 0
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
