"""Planted mistakes in the oracle are caught by its pins.

Each mutant changes one step of oracle/sq_oracle.c the way a plausible slip
would: a wrong operation, sign, constant, rounding rule, index or operand,
or a dropped term or clamp. The mutant is compiled with gcc on the CPU into
a scratch directory, and the pins of tests/test_oracle_pins.py are run
against it in this process. At least one pin must fail. The unchanged
source, compiled the same way, must fail none. No mutant reads or writes
outside its buffers, and the GPU path is not involved.
"""
import importlib.util
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")
SRC = os.path.join(ORACLE_DIR, "sq_oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (name, text in sq_oracle.c -- must occur exactly once, replacement)
MUTANTS = [
    ("act_smoothing_multiplies",
     "static float smooth_x(float v, float s_k) { return v / s_k; }",
     "static float smooth_x(float v, float s_k) { return v * s_k; }"),
    ("weight_smoothing_divides",
     "static float smooth_w(float v, float s_k) { return s_k * v; }",
     "static float smooth_w(float v, float s_k) { return v / s_k; }"),
    ("int8_rounds_half_away_from_zero",
     "float r = nearbyintf(v / scale);", "float r = roundf(v / scale);"),
    ("int8_truncates", "float r = nearbyintf(v / scale);", "float r = truncf(v / scale);"),
    ("int8_clamp_admits_minus_128",
     "if (r < -127.0f) r = -127.0f;", "if (r < -128.0f) r = -128.0f;"),
    ("int8_clamp_dropped", "    if (r > 127.0f) r = 127.0f;\n", "\n"),
    ("alpha_and_one_minus_alpha_swapped",
     "s[k] = (float)(pow(ax, alpha) / pow(aw, 1.0 - alpha));",
     "s[k] = (float)(pow(ax, 1.0 - alpha) / pow(aw, alpha));"),
    ("smoothing_factor_inverted",
     "s[k] = (float)(pow(ax, alpha) / pow(aw, 1.0 - alpha));",
     "s[k] = (float)(pow(aw, 1.0 - alpha) / pow(ax, alpha));"),
    ("epsilon_clamp_dropped",
     "double ax = (double)amax_x[k] > eps ? (double)amax_x[k] : eps;",
     "double ax = (double)amax_x[k];"),
    ("epsilon_too_small", "const double eps = 1e-5;", "const double eps = 1e-6;"),
    ("weight_epsilon_clamp_dropped",
     "double aw = (double)amax_w[k] > eps ? (double)amax_w[k] : eps;",
     "double aw = (double)amax_w[k];"),
    ("column_amax_without_abs",
     "float a = fabsf(load_elem(x, dtype, r * cols + c));\n                if (a > out[c])",
     "float a = load_elem(x, dtype, r * cols + c);\n                if (a > out[c])"),
    ("row_amax_without_abs",
     "float a = fabsf(load_elem(x, dtype, r * cols + c));\n                if (a > m)",
     "float a = load_elem(x, dtype, r * cols + c);\n                if (a > m)"),
    ("weight_scale_from_unsmoothed_amax",
     "float wt = s ? smooth_w(v, s[k]) : v;\n                float a = fabsf(wt);",
     "float wt = s ? smooth_w(v, s[k]) : v;\n                float a = fabsf(v);"),
    ("weight_e4m3_scale_uses_127",
     "    const float qmax = (qtype == 1) ? 448.0f : 127.0f;\n    /* Each thread",
     "    const float qmax = 127.0f;\n    /* Each thread"),
    ("weight_codes_not_transposed",
     "((int8_t*)wq)[n * K + k] =\n                        (scale == 0.0f) ? 0 : quant_i8(wt, scale);",
     "((int8_t*)wq)[k * N + n] =\n                        (scale == 0.0f) ? 0 : quant_i8(wt, scale);"),
    ("act_amax_without_abs",
     "float a = fabsf(xs);\n            if (a > amax) amax = a;\n        }\n        float scale = amax / qmax;",
     "float a = xs;\n            if (a > amax) amax = a;\n        }\n        float scale = amax / qmax;"),
    ("act_scale_divides_by_128",
     "float scale = amax / qmax;\n        sx[m] = scale;",
     "float scale = amax / (qmax + 1.0f);\n        sx[m] = scale;"),
    ("act_zero_row_not_special",
     "((int8_t*)xq)[m * K + k] =\n                    (scale == 0.0f) ? 0 : quant_i8(xs, scale);\n            }\n        }\n    }\n}\n\n/* -",
     "((int8_t*)xq)[m * K + k] =\n                    quant_i8(xs, scale);\n            }\n        }\n    }\n}\n\n/* -"),
    ("per_tensor_ignores_the_delayed_scale",
     "const float scale = scale_in ? *scale_in : amax / qmax;",
     "const float scale = amax / qmax;"),
    ("per_tensor_max_with_wrong_channel",
     "float xs = s ? smooth_x(v, s[i % K]) : v;", "float xs = s ? smooth_x(v, s[i / M]) : v;"),
    ("int8_gemm_drops_the_last_term",
     "for (int64_t k = 0; k < K; ++k)\n                a += (int32_t)xq",
     "for (int64_t k = 0; k + 1 < K; ++k)\n                a += (int32_t)xq"),
    ("int8_gemm_wrong_sign",
     "a += (int32_t)xq[m * K + k] * (int32_t)wq[n * K + k];",
     "a -= (int32_t)xq[m * K + k] * (int32_t)wq[n * K + k];"),
    ("e4m3_gemm_uses_x_twice",
     "a += table[xq[m * K + k]] * table[wq[n * K + k]];",
     "a += table[xq[m * K + k]] * table[xq[m * K + k]];"),
    ("sampled_int8_output_wrong_sign",
     "d += (int32_t)xr[k] * (int32_t)wr[k];", "d -= (int32_t)xr[k] * (int32_t)wr[k];"),
    ("sampled_e4m3_output_uses_w_twice",
     "for (int64_t k = 0; k < K; ++k) d += table[xr[k]] * table[wr[k]];",
     "for (int64_t k = 0; k < K; ++k) d += table[wr[k]] * table[wr[k]];"),
    ("epilogue_drops_the_bias",
     "if (has_bias) t = t + sqo_bf16_to_f32(bias_bf16);", "if (has_bias) t = t + 0.0f;"),
    ("epilogue_skips_the_channel_scale", "    t = t * sw_n;\n", "\n"),
    ("bf16_ties_away_from_zero",
     "if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;",
     "if (dropped >= 0x8000u) kept += 1u;"),
    ("bf16_truncates",
     "if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;",
     "(void)dropped;"),
    ("e4m3_ties_round_up", "else code = (lo % 2 == 0) ? lo : hi;", "else code = hi;"),
    ("e4m3_saturates_to_nan_code",
     "if (a >= 448.0) return (uint8_t)(sign | 0x7E);",
     "if (a >= 448.0) return (uint8_t)(sign | 0x7F);"),
    ("e4m3_subnormal_step_wrong",
     "ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    ("e4m3_exponent_bias_wrong",
     "ldexp((double)(8 + m), e - 10)", "ldexp((double)(8 + m), e - 11)"),
    ("column_amax_starts_at_one",
     "for (int64_t c = 0; c < cols; ++c) out[c] = 0.0f;",
     "for (int64_t c = 0; c < cols; ++c) out[c] = 1.0f;"),
    ("act_e4m3_codes_multiply_by_the_scale",
     "float scale = amax / qmax;\n        sx[m] = scale;\n        for (int64_t k = 0; k < K; ++k) {\n            float v = load_elem(x, dtype, m * K + k);\n            float xs = s ? smooth_x(v, s[k]) : v;\n            if (qtype == 1) {\n                ((uint8_t*)xq)[m * K + k] =\n                    (scale == 0.0f) ? 0 : sqo_e4m3_encode_rn_sat(xs / scale);",
     "float scale = amax / qmax;\n        sx[m] = scale;\n        for (int64_t k = 0; k < K; ++k) {\n            float v = load_elem(x, dtype, m * K + k);\n            float xs = s ? smooth_x(v, s[k]) : v;\n            if (qtype == 1) {\n                ((uint8_t*)xq)[m * K + k] =\n                    (scale == 0.0f) ? 0 : sqo_e4m3_encode_rn_sat(xs * scale);"),
    ("weight_e4m3_codes_unscaled",
     "(scale == 0.0f) ? 0 : sqo_e4m3_encode_rn_sat(wt / scale);",
     "(scale == 0.0f) ? 0 : sqo_e4m3_encode_rn_sat(wt);"),
    ("e4m3_sign_dropped",
     "uint8_t sign = signbit(x) ? 0x80 : 0x00;", "uint8_t sign = 0x00;"),
    ("per_tensor_max_of_unsmoothed_values",
     "float a = fabsf(xs);\n        if (a > amax) amax = a;\n    }\n    *amax_out = amax;",
     "float a = fabsf(v);\n        if (a > amax) amax = a;\n    }\n    *amax_out = amax;"),
    ("per_tensor_reports_the_scale_as_max",
     "*amax_out = amax;", "*amax_out = amax / qmax;"),
    ("bf16_widening_shifted_wrong",
     "return bits_f32((uint32_t)h << 16);", "return bits_f32((uint32_t)h << 15);"),
    ("fold_reads_the_transpose",
     "smooth_x(load_elem(p, dtype, r * cols + c),", "smooth_x(load_elem(p, dtype, c * rows + r),"),
    ("fold_multiplies",
     "out[r * cols + c] = smooth_x(load_elem(p, dtype, r * cols + c),",
     "out[r * cols + c] = smooth_w(load_elem(p, dtype, r * cols + c),"),
    ("fold_ignores_the_axis",
     "per_column ? s[c] : s[r]);", "s[c < r ? c : r]);"),
    ("int4_scale_divides_by_8", "float scale = amax / 7.0f;", "float scale = amax / 8.0f;"),
    ("int4_truncates",
     "float c = nearbyintf(v / scale);", "float c = truncf(v / scale);"),
    ("int4_even_and_odd_halves_swapped",
     "static int nibble_shift(int64_t k) { return (int)((k & 1) ? 16 + 4 * ((k & 7) >> 1) : 4 * ((k & 7) >> 1)); }",
     "static int nibble_shift(int64_t k) { return (int)((k & 1) ? 4 * ((k & 7) >> 1) : 16 + 4 * ((k & 7) >> 1)); }"),
    ("int4_word_bytes_big_endian",
     "for (int b = 0; b < 4; ++b) row[4 * g + b] = (uint8_t)(word >> (8 * b));",
     "for (int b = 0; b < 4; ++b) row[4 * g + b] = (uint8_t)(word >> (24 - 8 * b));"),
    ("int4_nibble_not_sign_extended",
     "return (int8_t)((nb & 0x08u) ? (int)nb - 16 : (int)nb);", "return (int8_t)nb;"),
    ("weight_only_drops_the_scale",
     "double w_deq = (double)q * (double)sw[n];", "double w_deq = (double)q;"),
    ("weight_only_drops_the_bias",
     "if (bias) acc += (double)sqo_bf16_to_f32(bias[n]);", "(void)bias;"),
    ("weight_only_reads_the_wrong_code",
     "q = unpack_code((const uint8_t*)wq + n * (K / 2), k);",
     "q = unpack_code((const uint8_t*)wq + n * (K / 2), k ^ 1);"),
    ("weight_only_wrong_channel_scale",
     "double w_deq = (double)q * (double)sw[n];", "double w_deq = (double)q * (double)sw[m % N];"),
    ("rms_drops_eps", "const double v = mean + (double)eps;", "const double v = mean;"),
    ("rms_divides_by_k_minus_one", "const double mean = ss / (double)K;",
     "const double mean = ss / (double)(K - 1);"),
    ("rms_square_window_off_by_one", "<< (2 * (e - emax) + 96);", "<< (2 * (e - emax) + 95);"),
    ("rms_no_square_root", "const double t = sqrt(v);", "const double t = v;"),
    ("rms_no_reciprocal", "const float r = (float)(1.0 / t);", "const float r = (float)t;"),
    ("rms_gain_before_the_norm", "const float a = sqo_bf16_to_f32(xk) * r;\n    return a * gk;",
     "const float a = sqo_bf16_to_f32(xk) * gk;\n    return a * r;"),
    ("rms_binary32_root", "const float r = (float)(1.0 / t);",
     "const float r = 1.0f / sqrtf((float)v);"),
]


def _compile(src_text, tmp_path, name):
    c_file = tmp_path / f"{name}.c"
    c_file.write_text(src_text)
    so = tmp_path / f"lib_{name}.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                    "-fPIC", "-shared", "-Wno-unused-variable", "-I", ORACLE_DIR, "-o", str(so),
                    str(c_file), "-lm"], check=True)
    return str(so)


def _oracle_on(so, name):
    """A fresh copy of the oracle's Python binding bound to the library `so`."""
    spec = importlib.util.spec_from_file_location(f"oracle_{name}",
                                                  os.path.join(ORACLE_DIR, "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._LIB = so
    mod.build = lambda force=False: so
    return mod


def _pins_with(oracle_mod, name):
    """The pin module executed with `import oracle` resolving to oracle_mod."""
    saved = sys.modules.get("oracle")
    sys.modules["oracle"] = oracle_mod
    try:
        spec = importlib.util.spec_from_file_location(f"pins_{name}", PINS)
        pins = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(pins)
    finally:
        if saved is None:
            sys.modules.pop("oracle", None)
        else:
            sys.modules["oracle"] = saved
    return pins


def _cases(pins):
    for fname, f in sorted(vars(pins).items()):
        if not (fname.startswith("test_") and callable(f)):
            continue
        params = [m for m in getattr(f, "pytestmark", []) if m.name == "parametrize"]
        if not params:
            yield fname, f, {}
            continue
        assert len(params) == 1, fname
        argnames, values = params[0].args[0], params[0].args[1]
        names = [a.strip() for a in argnames.split(",")]
        for v in values:
            yield fname, f, dict(zip(names, v if len(names) > 1 else (v,)))


def _failing_pins(pins):
    failed = []
    for fname, f, kw in _cases(pins):
        try:
            f(**kw)
        except Exception:  # noqa: BLE001 - any failure of a pin counts
            failed.append(fname)
    return failed


def test_unmutated_oracle_passes_every_pin(tmp_path):
    so = _compile(open(SRC).read(), tmp_path, "unmutated")
    pins = _pins_with(_oracle_on(so, "unmutated"), "unmutated")
    assert sum(1 for _ in _cases(pins)) >= 45
    assert _failing_pins(pins) == []


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site is not unique: {old!r}"
    so = _compile(src.replace(old, new), tmp_path, name)
    failed = _failing_pins(_pins_with(_oracle_on(so, name), name))
    assert failed, f"no pin caught the planted mistake {name}"
