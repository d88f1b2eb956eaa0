"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a temporary copy of the oracle's C source (a
swapped operand, a wrong sign, a dropped term, an off-by-one, a wrong
rounding), builds it, and runs the CPU pin suite against it in a subprocess:
the suite must fail. Nothing here touches the committed oracle or a GPU.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "echo_oracle.c")

MUTANTS = {
    "swap_ema_in_compensation": [("float t1 = w * e_short;", "float t1 = w * e_long;"),
                                 ("float t2 = one_minus_w * e_long;", "float t2 = one_minus_w * e_short;")],
    "one_minus_w_dropped": [("float one_minus_w = 1.0f - w;", "float one_minus_w = w;")],
    "residual_sign": [("res[base + (size_t)i] = xp[base + (size_t)i] - vhat[i];",
                       "res[base + (size_t)i] = vhat[i] - xp[base + (size_t)i];")],
    "owner_residual_sign": [("res[obase + (size_t)i] = sum[i] - oracle_bf16_to_f32(y_owner[i]);",
                             "res[obase + (size_t)i] = oracle_bf16_to_f32(y_owner[i]) - sum[i];")],
    "ema_drops_memory": [("        e[i] = u + v;", "        e[i] = v;")],
    "ema_rates_swapped": [("oracle_ema_update(&e_long[base], &res[base], m, alpha_long);",
                           "oracle_ema_update(&e_long[base], &res[base], m, alpha_short);")],
    "owner_term_quantized": [("            if (r == o) {\n                for (int i = 0; i < m; i++) {\n                    vtmp[i] = xp[base + (size_t)i];",
                              "            if (r == o && 0) {\n                for (int i = 0; i < m; i++) {\n                    vtmp[i] = xp[base + (size_t)i];"),
                             ("            if (r == o) {\n                continue;\n            }",
                              "            if (0) {\n                continue;\n            }")],
    "sum_drops_a_term": [("                    sum[i] = sum[i] + vtmp[i];", "                    sum[i] = vtmp[i];")],
    "nibbles_swapped": [("out[i] = (uint8_t)(lo | (hi << 4));", "out[i] = (uint8_t)(hi | (lo << 4));"),
                        ("codes[2 * i] = (uint8_t)(packed[i] & 0xF);\n        codes[2 * i + 1] = (uint8_t)(packed[i] >> 4);",
                         "codes[2 * i + 1] = (uint8_t)(packed[i] & 0xF);\n        codes[2 * i] = (uint8_t)(packed[i] >> 4);")],
    "zero_rounded_to_nearest": [("zh = oracle_f32_to_f16(mn, ORACLE_RD);",
                                 "zh = oracle_f32_to_f16(mn, ORACLE_RN);")],
    "scale_rounded_down": [("float d = mx - zd;\n        float step = d / (float)Q;\n        sh = oracle_f32_to_f16(step, ORACLE_RU);",
                            "float d = mx - zd;\n        float step = d / (float)Q;\n        sh = oracle_f32_to_f16(step, ORACLE_RD);")],
    # the quantizer forms of the ablations
    "nearest_zero_rounded_down": [("zh = oracle_f32_to_f16(mn, ORACLE_RN);", "zh = oracle_f32_to_f16(mn, ORACLE_RD);")],
    "nearest_scale_rounded_up": [("sh = oracle_f32_to_f16(step, ORACLE_RN);", "sh = oracle_f32_to_f16(step, ORACLE_RU);")],
    "nearest_scale_from_rounded_zero": [("        float d = mx - mn;\n", "        float d = mx - oracle_f16_to_f32(zh);\n")],
    "codes_not_clamped_above": [("    if (c > Q) {\n        c = Q;\n    }\n", "")],
    "int_zero_scale_rounded_down": [("uint16_t sh = oracle_f32_to_f16(step, ORACLE_RU);",
                                     "uint16_t sh = oracle_f32_to_f16(step, ORACLE_RD);")],
    "int_zero_range_not_widened": [("float lo = mn < 0.0f ? mn : 0.0f;", "float lo = mn;")],
    "int_zero_point_sign": [("float nlo = -lo;", "float nlo = lo;")],
    "int_zero_codes_without_zero_point": [("c = round_clamp(u, zp, Q);", "c = round_clamp(u, 0, Q);")],
    "int_zero_dequant_drops_zero_point": [("        int k = code - (int)z_bits;", "        int k = code;")],
    "codes_truncated": [("float r = rintf(u);", "float r = floorf(u);")],
    "segment_off_by_one": [("if (j >= oracle_segment_begin(s, G, P) && j < oracle_segment_begin(s + 1, G, P)) {",
                            "if (j >= oracle_segment_begin(s, G, P) && j <= oracle_segment_begin(s + 1, G, P)) {")],
    "ties_not_even": [("k = (fmod(lo, 2.0) == 0.0) ? lo : hi;", "k = hi;")],
    "no_minus_zero_fix": [("    mn = mn + 0.0f;\n    mx = mx + 0.0f;\n", "")],
    "no_feedback_add": [("                xp[idx] = xv + c;", "                xp[idx] = xv;")],
    # evaluation orders: the owner's sum in rank order, the EMA as (1 - a) e + a rho
    "sum_reverse_order": [("        for (int r = 0; r < P; r++) {\n            size_t base = (size_t)r * (size_t)ld + (size_t)(jl * group);\n            if (r == o) {",
                           "        for (int r = P - 1; r >= 0; r--) {\n            size_t base = (size_t)r * (size_t)ld + (size_t)(jl * group);\n            if (r == o) {"),
                          ("                if (r == 0) {\n                    sum[i] = vtmp[i];",
                           "                if (r == P - 1) {\n                    sum[i] = vtmp[i];")],
    "sum_owner_first": [("        for (int r = 0; r < P; r++) {\n            size_t base = (size_t)r * (size_t)ld + (size_t)(jl * group);\n            if (r == o) {",
                         "        for (int rr = 0; rr < P; rr++) {\n            int r = (o + rr) % P;\n            size_t base = (size_t)r * (size_t)ld + (size_t)(jl * group);\n            if (r == o) {"),
                        ("                if (r == 0) {\n                    sum[i] = vtmp[i];",
                         "                if (rr == 0) {\n                    sum[i] = vtmp[i];")],
    "sum_owner_last": [("        for (int r = 0; r < P; r++) {\n            size_t base = (size_t)r * (size_t)ld + (size_t)(jl * group);\n            if (r == o) {",
                        "        for (int rr = 0; rr < P; rr++) {\n            int r = (o + 1 + rr) % P;\n            size_t base = (size_t)r * (size_t)ld + (size_t)(jl * group);\n            if (r == o) {"),
                       ("                if (r == 0) {\n                    sum[i] = vtmp[i];",
                        "                if (rr == 0) {\n                    sum[i] = vtmp[i];")],
    "bf16_baseline_reverse_order": [("        for (int r = 0; r < P; r++) {\n            float v = oracle_bf16_to_f32(x[(size_t)r * (size_t)n + (size_t)i]);\n            if (r == 0) {",
                                     "        for (int r = P - 1; r >= 0; r--) {\n            float v = oracle_bf16_to_f32(x[(size_t)r * (size_t)n + (size_t)i]);\n            if (r == P - 1) {")],
    "bf16_baseline_drops_a_rank": [("            float v = oracle_bf16_to_f32(x[(size_t)r * (size_t)n + (size_t)i]);\n            if (r == 0) {",
                                    "            float v = r == P - 1 && P > 1 ? 0.0f : oracle_bf16_to_f32(x[(size_t)r * (size_t)n + (size_t)i]);\n            if (r == 0) {")],
    "ema_incremental_form": [("        float u = keep * e[i];\n        float v = alpha * rho[i];\n        e[i] = u + v;",
                              "        float d = rho[i] - e[i];\n        float v = alpha * d;\n        e[i] = e[i] + v;\n        (void)keep;")],
}

PIN_FILES = ["tests/test_oracle_order.py", "tests/test_oracle_bf16.py", "tests/test_oracle_call.py", "tests/test_oracle_quantizer.py", "tests/test_oracle_variants.py",
             "tests/test_oracle_chain.py", "tests/test_oracle_convert.py"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    with open(SRC) as f:
        src = f.read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, f"mutation site not found once: {old!r}"
        src = src.replace(old, new)
    csrc = tmp_path / "mutant.c"
    lib = tmp_path / "libmutant.so"
    csrc.write_text(src)
    subprocess.run(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-frounding-math",
                    "-fPIC", "-shared", str(csrc), "-o", str(lib), "-lm"], check=True)
    env = dict(os.environ, ECHO_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PIN_FILES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
