"""Plant plausible mistakes in copies of the CPU oracle and check that the
pins catch every one of them (mutation testing, CPU only).

Each mutant is the oracle's C source with one textual change, compiled to a
temporary shared library.  A mutant "survives" if every pin still passes.
"""
import os
import tempfile

import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins

MUTANTS = {
    # quantization
    "scale_over_128": ("amax / 127.0f", "amax / 128.0f"),
    "round_half_away": ("nearbyintf(r)", "roundf(r)"),
    "truncate": ("nearbyintf(r)", "truncf(r)"),
    "divide_by_fp32_scale": ("float r = col_vals[k] / s;", "float r = col_vals[k] / s32;"),
    "clip_to_minus_128": ("if (rr < -127.0f) {\n                rr = -127.0f;",
                          "if (rr < -128.0f) {\n                rr = -128.0f;"),
    "no_abs_in_bound": ("float a = fabsf(col_vals[k]);", "float a = col_vals[k];"),
    "bound_skips_first_row": ("    for (int64_t k = 0; k < K; ++k) {\n        float a",
                              "    for (int64_t k = 1; k < K; ++k) {\n        float a"),
    # fp16 codec
    "f16_ties_away": ("(rem == half && (q & 1ull))", "(rem == half)"),
    "f16_flush_subnormals": ("    return (uint16_t)(sign | (uint32_t)M);\n}",
                             "    return (uint16_t)(sign);\n}"),
    "f16_exponent_off_by_one": ("int32_t biased = E + 25;", "int32_t biased = E + 24;"),
    # linear
    "drop_scale": ("double y = acc[n] * (double)oracle_f16_to_f32(scales[n]);",
                   "double y = acc[n];"),
    "bias_subtracted": ("y += (double)oracle_f16_to_f32(bias[n]);",
                        "y -= (double)oracle_f16_to_f32(bias[n]);"),
    "transposed_weight_index": ("acc[n] += x * (double)qrow[n];",
                                "acc[n] += x * (double)q[n * K + k];"),
    "x_row_ignored": ("oracle_f16_to_f32(X[m * K + k])", "oracle_f16_to_f32(X[k])"),
    "scale_indexed_by_row": ("(double)oracle_f16_to_f32(scales[n]);",
                             "(double)oracle_f16_to_f32(scales[m]);"),
    # asymmetric quantization
    "asym_256_levels": ("range / 255.0f", "range / 256.0f"),
    "asym_zero_point_sign": ("nearbyintf(-128.0f - t)", "nearbyintf(-128.0f + t)"),
    "asym_range_without_zero": ("float lo = 0.0f, hi = 0.0f;", "float lo = col_vals[0], hi = col_vals[0];"),
    "asym_zero_point_not_added": ("qi = (int32_t)rr + z;", "qi = (int32_t)rr;"),
    "asym_clip_at_minus_127": ("if (qi < -128) {\n                qi = -128;", "if (qi < -127) {\n                qi = -127;"),
    "asym_linear_zero_point_dropped": ("(double)((int32_t)codes[col] - (int32_t)zeros[col])", "(double)codes[col]"),
    "asym_linear_zero_point_added": ("(double)((int32_t)codes[col] - (int32_t)zeros[col])",
                                     "(double)((int32_t)codes[col] + (int32_t)zeros[col])"),
    # clipped scale
    "percentile_rank_off_by_one": ("bound = sort_buf[r - 1];", "bound = sort_buf[r > 1 ? r - 2 : 0];"),
    "percentile_floor_rank": ("double rr = ceil(param * (double)K);", "double rr = floor(param * (double)K);"),
    "percentile_signed_values": ("sort_buf[k] = fabsf(col_vals[k]);", "sort_buf[k] = col_vals[k];"),
    "fixed_clip_ignored": ("if (bound > cf) {", "if (0) {"),
    "fixed_clip_param_rounded_down": ("float cf = (float)param;",
                                      "float cf = (float)param; if ((double)cf > param) cf = nextafterf(cf, 0.0f);"),
    "clip_codes_not_clamped": ("rr = clampf_range(rr, -127.0f, 127.0f);", "rr = clampf_range(rr, -128.0f, 127.0f);"),
    # outlier split
    "outlier_at_or_above_bound": ("if (fabsf(col_buf[k]) > cut && c < cap) {",
                                  "if (fabsf(col_buf[k]) >= cut && c < cap) {"),
    "outlier_code_kept": ("                q[k * N + n] = 0;\n", ""),
    "outlier_value_not_added": ("            Y[m * N + n] += extra;", "            Y[m * N + n] += 0.0 * extra;"),
    "outlier_row_as_token": ("X[m * K + rows[n * cap + j]]", "X[rows[n * cap + j] % M * K + m % K]"),
    "outlier_value_fp32_truncated": ("vals[n * cap + c] = oracle_f32_to_f16(col_buf[k]);",
                                     "vals[n * cap + c] = (uint16_t)(oracle_f32_to_f16(col_buf[k]) & 0xFFFCu);"),
    "asym_linear_scale_by_row": ("acc[col] * (double)oracle_f16_to_f32(scales[col])",
                                 "acc[col] * (double)oracle_f16_to_f32(scales[row])"),
    # fp16 widening
    "f16_subnormal_step_halved": ("mag = ldexpf((float)frac, -24);", "mag = ldexpf((float)frac, -25);"),
    "f16_normal_bias_off_by_one": ("(int)exp - 25);", "(int)exp - 24);"),
    # more of the variants
    "outlier_rows_descending": ("        for (int64_t k = 0; k < K; ++k) {\n            /* at most K - r",
                                "        for (int64_t k = K - 1; k >= 0; --k) {\n            /* at most K - r"),
    "asym_divide_by_fp32_scale": ("float rr = nearbyintf(col_vals[k] / s);\n            /* |W / S| stays",
                                  "float rr = nearbyintf(col_vals[k] / (range / 255.0f));\n            /* |W / S| stays"),
    "asym_zero_point_from_max": ("float t = lo / s;", "float t = hi / s;"),
    # clamp and GEMM details
    "clamp_top_at_128": ("            if (rr > 127.0f) {\n                rr = 127.0f;\n            }\n            if (rr < -127.0f) {",
                         "            if (rr > 128.0f) {\n                rr = 128.0f;\n            }\n            if (rr < -127.0f) {"),
    "linear_fp32_accumulation": ("                acc[n] += x * (double)qrow[n];",
                                 "                acc[n] = (double)(float)(acc[n] + x * (double)qrow[n]);"),
    "bias_scaled": ("                y += (double)oracle_f16_to_f32(bias[n]);\n            }\n            Y[m * N + n] = y;\n        }\n    }\n}\n\n/* ------",
                    "                y += (double)oracle_f16_to_f32(bias[n]) * (double)oracle_f16_to_f32(scales[n]);\n            }\n            Y[m * N + n] = y;\n        }\n    }\n}\n\n/* ------"),
}


def _compile_mutant(name, old, new, tmpdir):
    with open(oracle._SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/found"
    path = os.path.join(tmpdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(tmpdir, f"lib{name}.so")
    oracle.build(force=True, src=path, out=so)
    return oracle.Oracle(so)


@pytest.fixture(scope="module")
def tmpdir():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_kill_mutant(name, tmpdir):
    old, new = MUTANTS[name]
    orc = _compile_mutant(name, old, new, tmpdir)
    killed = []
    for pin in pins.PINS:
        try:
            with np.errstate(all="ignore"):
                pin(orc)
        except (AssertionError, ValueError, IndexError):
            killed.append(pin.__name__)
    assert killed, f"mutant {name} survived every pin"
