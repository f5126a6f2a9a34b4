"""The oracle's pins must be able to fail.

Each case below plants one plausible mistake in a copy of the oracle's C
source (a dropped term, a wrong sign or index, a transposed operand, a
changed range or rounding rule), builds that copy, and runs the oracle pin
suite (``test_oracle.py``) against it in a child process.  Every broken copy
has to fail at least one pin; the unbroken copy, built the same way, has to
pass them all.  The planted mistakes live only in temporary copies on the
CPU.

Passages the mistakes contradict: "QServe: W4A8KV4 Quantization and System
Co-design for Efficient LLM Serving" (velog notes), Methods 1) Algorithm: QoQ
(per-channel INT8 first level, per-group UINT4 second level) and 2) System:
QServe (protective range, dq = q*s2 - z*s2); same page, Background (the
scaling applied once, after the K reduction); IEEE 754 binary16 for the
FP16 conversions.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "qoq_oracle.c")

# (name, text in qoq_oracle.c, replacement).  Each text occurs exactly once.
MUTANTS = [
    # FP16 decode / encode
    ("h2d_subnormal_exponent",
     "ldexp((double)f, -24)", "ldexp((double)f, -25)"),
    ("h2d_exponent_bias",
     "ldexp((double)(1024 + f), e - 25)", "ldexp((double)(1024 + f), e - 24)"),
    ("h2d_drops_sign",
     "return sign ? -v : v;", "return v;"),
    ("d2h_ties_round_down",
     "if (diff < 0.5) return fl;", "if (diff <= 0.5) return fl;"),
    ("d2h_ties_away_from_zero",
     "return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;", "return fl + 1.0;"),
    ("d2h_overflow_threshold",
     "if (a >= 65520.0) return sign | 0x7c00;",
     "if (a > 65504.0) return sign | 0x7c00;"),
    ("d2h_subnormal_quantum",
     "double n = round_half_even_d(ldexp(a, 24));",
     "double n = round_half_even_d(ldexp(a, 23));"),
    ("d2h_mantissa_carry_lost",
     "if (n == 2048.0) { n = 1024.0; e += 1; }", "if (n == 2048.0) { n = 1024.0; }"),
    # integer round-half-even division
    ("rne_div_ties_up",
     "if (twice > b || (twice == b && (q & 1))) {", "if (twice >= b) {"),
    ("rne_div_truncates",
     "q += (a < 0) ? -1 : 1;", "q += 0;"),
    ("rne_div_wrong_direction_for_negatives",
     "q += (a < 0) ? -1 : 1;", "q += 1;"),
    ("h2d_infinity_is_nan",
     "v = f ? NAN : INFINITY;", "v = NAN;"),
    ("d2h_nan_is_infinity",
     "if (isnan(x)) return 0x7e00;", "if (isnan(x)) return 0x7c00;"),
    ("rne_f_ties_away",
     "static float rne_f(float v) { return rintf(v); }",
     "static float rne_f(float v) { return roundf(v); }"),
    # scales
    ("scale_zero_guard_missing",
     "if ((s & 0x7fff) == 0) s = 0x0001;", "if ((s & 0x7fff) == 0) s = 0x0000;"),
    ("scale_all_zero_row_is_two",
     "if (amax == 0.0f) return 0x3c00;", "if (amax == 0.0f) return 0x4000;"),
    # level 1
    ("level1_range_127",
     "uint16_t s = scale_from_absmax(amax, (float)ORC_R1);",
     "uint16_t s = scale_from_absmax(amax, 127.0f);"),
    ("level1_no_clamp",
     "W8[(size_t)n * K + k] = (int8_t)clampi(v, -ORC_R1, ORC_R1);",
     "W8[(size_t)n * K + k] = (int8_t)v;"),
    ("level1_signed_max",
     "float v = fabsf(orc_h2f(row[k]));\n            if (v > amax) amax = v;\n        }\n"
     "        uint16_t s = scale_from_absmax(amax, (float)ORC_R1);",
     "float v = orc_h2f(row[k]);\n            if (v > amax) amax = v;\n        }\n"
     "        uint16_t s = scale_from_absmax(amax, (float)ORC_R1);"),
    ("level1_unrounded_scale",
     "float sf = orc_h2f(s);\n        for (int k = 0; k < K; ++k) {\n"
     "            float t = orc_h2f(row[k]) / sf;",
     "float sf = amax / (float)ORC_R1;\n        for (int k = 0; k < K; ++k) {\n"
     "            float t = orc_h2f(row[k]) / sf;"),
    ("level1_truncates",
     "int v = (int)rne_f(t);", "int v = (int)t;"),
    # level 2
    ("level2_scale_floor",
     "int s = (range + 14) / 15;", "int s = range / 15;"),
    ("level2_scale_rounded_to_nearest",
     "int s = (range + 14) / 15;", "int s = (range + 7) / 15;"),
    ("level2_range_excludes_zero",
     "int mn = 0, mx = 0;", "int mn = 127, mx = -128;"),
    ("level2_zero_sign",
     "int zz = orc_rne_div(-mn, s);", "int zz = orc_rne_div(mn, s);"),
    ("level2_zero_truncated",
     "int zz = orc_rne_div(-mn, s);", "int zz = -mn / s;"),
    ("level2_zero_point_dropped_from_code",
     "int c = orc_rne_div(w[i], s) + zz;", "int c = orc_rne_div(w[i], s);"),
    ("level2_code_clamp_14",
     "(uint8_t)clampi(c, 0, 15);", "(uint8_t)clampi(c, 0, 14);"),
    ("level2_max_ignored",
     "if (w[i] > mx) mx = w[i];", "(void)mx;"),
    ("level2_group_offset_dropped",
     "const int8_t* w = W8 + (size_t)n * K + (size_t)g * G;",
     "const int8_t* w = W8 + (size_t)n * K;"),
    # dequantization dq = q*s2 - z*s2
    ("dequant_drops_zero_term",
     "int v = (int)q[(size_t)n * K + k] * s - zz * s;",
     "int v = (int)q[(size_t)n * K + k] * s;"),
    ("dequant_adds_zero_term",
     "int v = (int)q[(size_t)n * K + k] * s - zz * s;",
     "int v = (int)q[(size_t)n * K + k] * s + zz * s;"),
    ("dequant_drops_scale",
     "int v = (int)q[(size_t)n * K + k] * s - zz * s;",
     "int v = (int)q[(size_t)n * K + k] - zz;"),
    ("dequant_group_of_next_channel",
     "int s = s2[(size_t)n * ng + k / G];", "int s = s2[(size_t)n * ng + (k / G + 1) % ng];"),
    # activations
    ("act_range_119",
     "uint16_t s = scale_from_absmax(amax, (float)ORC_QMAX_X);",
     "uint16_t s = scale_from_absmax(amax, (float)ORC_R1);"),
    ("act_clamp_128",
     "clampi(v, -ORC_QMAX_X, ORC_QMAX_X)", "clampi(v, -128, ORC_QMAX_X)"),
    ("act_truncates",
     "int v = (int)rne_f(orc_h2f(row[k]) / sf);", "int v = (int)(orc_h2f(row[k]) / sf);"),
    # integer GEMM
    ("gemm_drops_first_term",
     "for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];",
     "for (int k = 1; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];"),
    ("gemm_reversed_operand",
     "for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];",
     "for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[K - 1 - k];"),
    ("gemm_overflow_unchecked",
     "if (s > INT32_MAX || s < INT32_MIN) overflow += 1;", "(void)0;"),
    ("gemm_sampled_positions_swapped",
     "out[i] = orc_dot_i8(X8 + (size_t)ms[i] * K, dq + (size_t)ns[i] * K, K);",
     "out[i] = orc_dot_i8(X8 + (size_t)ms[i] * K, dq + (size_t)ms[i] * K, K);"),
    # epilogue
    ("epilogue_transposed_accumulator",
     "double v = (double)acc[(size_t)m * N + n] * a * orc_h2d(s1[n]);",
     "double v = (double)acc[(size_t)n * M + m] * a * orc_h2d(s1[n]);"),
    ("epilogue_drops_channel_scale",
     "double v = (double)acc[(size_t)m * N + n] * a * orc_h2d(s1[n]);",
     "double v = (double)acc[(size_t)m * N + n] * a;"),
    ("epilogue_first_token_scale",
     "double a = orc_h2d(sx[m]);", "double a = orc_h2d(sx[0]);"),
    ("epilogue_single_precision",
     "double v = (double)acc[(size_t)m * N + n] * a * orc_h2d(s1[n]);",
     "double v = (double)((float)acc[(size_t)m * N + n] * (float)a"
     " * (float)orc_h2d(s1[n]));"),
    # per-input-channel smoothing
    ("smooth_strength_one",
     "float r = sqrtf(ax / aw);", "float r = ax / aw;"),
    ("smooth_factor_inverted",
     "float r = sqrtf(ax / aw);", "float r = sqrtf(aw / ax);"),
    ("smooth_zero_guard_zero",
     "s[k] = 0x3c00;                        /* 1.0 */", "s[k] = 0x0000;"),
    ("smooth_no_upper_clamp",
     "if (r > 0x1p14f) r = 0x1p14f;", "if (r > 0x1p20f) r = 0x1p20f;"),
    ("smooth_activations_multiplied",
     "orc_f2h(orc_h2f(X[(size_t)m * K + k]) / orc_h2f(s[k]))",
     "orc_f2h(orc_h2f(X[(size_t)m * K + k]) * orc_h2f(s[k]))"),
    ("smooth_weights_divided",
     "orc_d2h(orc_h2d(W[(size_t)n * K + k]) * orc_h2d(s[k]))",
     "orc_d2h(orc_h2d(W[(size_t)n * K + k]) / orc_h2d(s[k]))"),
    ("smooth_weights_rounded_twice",
     "orc_d2h(orc_h2d(W[(size_t)n * K + k]) * orc_h2d(s[k]))",
     "orc_f2h((float)orc_h2d(W[(size_t)n * K + k]) * (float)orc_h2d(s[k]) + 0x1p-30f)"),
    ("smooth_factor_row_max_of_weights",
     "float v = fabsf(orc_h2f(W[(size_t)n * K + k]));\n            if (v > aw) aw = v;",
     "float v = fabsf(orc_h2f(W[(size_t)n * K + (k % N)]));\n            if (v > aw) aw = v;"),
    # SiLU(gate) * up
    ("silu_is_sigmoid",
     "double silu = g / (1.0 + exp(-g));", "double silu = 1.0 / (1.0 + exp(-g));"),
    ("silu_exponent_sign",
     "double silu = g / (1.0 + exp(-g));", "double silu = g / (1.0 + exp(g));"),
    ("silu_gate_and_up_swapped",
     "double g = orc_h2d(G[i]);", "double g = orc_h2d(U[i]);"),
    ("silu_without_up",
     "H[i] = orc_d2h(silu * orc_h2d(U[i]));", "H[i] = orc_d2h(silu);"),
    # 4-bit KV cache and decode attention
    ("kv4_scale_over_16",
     "uint16_t sh = orc_f2h(range / 15.0f);", "uint16_t sh = orc_f2h(range / 16.0f);"),
    ("kv4_codes_truncated",
     "c = clampi((int)rne_f(t), 0, 15);", "c = clampi((int)t, 0, 15);"),
    ("kv4_codes_clamped_to_16",
     "c = clampi((int)rne_f(t), 0, 15);", "c = clampi((int)rne_f(t), 0, 16);"),
    ("kv4_offset_not_subtracted",
     "float t = (orc_h2f(x[i]) - mn) / sv;", "float t = orc_h2f(x[i]) / sv;"),
    ("kv4_dequant_drops_offset",
     "out[r * d + i] = sv * (double)q[r * d + i] + mv;", "out[r * d + i] = sv * (double)q[r * d + i];"),
    ("kv4_score_scaled_by_1_over_d",
     "score[t] = acc / sqrt((double)d);", "score[t] = acc / (double)d;"),
    ("kv4_grouped_heads_modulo",
     "const int hk = h / g;", "const int hk = h % Hkv;"),
    ("kv4_exponent_sign",
     "score[t] = exp(score[t] - mx);", "score[t] = exp(mx - score[t]);"),
    ("kv4_values_use_key_scales",
     "acc += score[t] * (orc_h2d(sv[r]) * (double)qv[r * d + i] + orc_h2d(mv[r]));",
     "acc += score[t] * (orc_h2d(sk[r]) * (double)qv[r * d + i] + orc_h2d(mv[r]));"),
    ("kv4_values_drop_offset",
     "acc += score[t] * (orc_h2d(sv[r]) * (double)qv[r * d + i] + orc_h2d(mv[r]));",
     "acc += score[t] * (orc_h2d(sv[r]) * (double)qv[r * d + i]);"),
    ("kv4_not_normalized_by_weights",
     "acc /= sum;", "acc /= (double)Lb;"),
]


def _source():
    with open(SRC, encoding="utf-8") as f:
        return f.read()


def test_each_mistake_names_one_place():
    src = _source()
    names = [m[0] for m in MUTANTS]
    assert len(names) == len(set(names))
    for name, old, new in MUTANTS:
        assert src.count(old) == 1, name
        assert old != new, name


def _run_pins(lib_path):
    env = dict(os.environ, QOQ_ORACLE_LIB=lib_path, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "pytest", os.path.join(HERE, "test_oracle.py"),
           "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return r.returncode, r.stdout[-2000:]


def _build_and_run(tmp_dir, name, text):
    src = os.path.join(tmp_dir, f"{name}.c")
    with open(src, "w", encoding="utf-8") as f:
        f.write(text)
    lib = oracle.compile_library(src, os.path.join(tmp_dir, f"lib{name}.so"))
    return _run_pins(lib)


def test_pins_catch_every_planted_mistake(tmp_path):
    src = _source()
    jobs = [("unchanged", src)] + [(n, src.replace(o, r)) for n, o, r in MUTANTS]
    workers = max(1, min(8, os.cpu_count() or 1))
    with ThreadPoolExecutor(workers) as ex:
        results = dict(zip(
            [j[0] for j in jobs],
            ex.map(lambda j: _build_and_run(str(tmp_path), j[0], j[1]), jobs)))
    rc, out = results.pop("unchanged")
    assert rc == 0, out
    survivors = [name for name, (rc, _) in results.items() if rc == 0]
    assert not survivors, f"pins did not catch: {survivors}"
    # a child that crashed instead of failing a pin would also give rc != 0;
    # require the ordinary pytest failure code
    crashed = {name: rc for name, (rc, _) in results.items() if rc != 1}
    assert not crashed, crashed
