"""Planted mistakes: each variant below copies the oracle's C source, injects one plausible
bug (a dropped term, a wrong tie rule, a transposed index, ...), builds it on the CPU and
runs the pin suite against it. Every variant must make the pins fail: this shows the pins
are strong enough to catch that class of mistake."""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "drop_h_weight": ("e += (double)cw[j] * (d * d);", "e += (d * d);"),
    "ties_always_up": ("return (lo % 2 == 0) ? lo : hi;", "return hi;"),
    "naive_divisor": ("return nearest_rne(T_E4M3, 127, amax / 6.0f);",
                      "return nearest_rne(T_E4M3, 127, amax / 4.0f);"),
    "candidate_ties_high": ("if (e < *e1) { *e2 = *e1; *e1 = e; *cbest = c; }",
                            "if (e <= *e1) { *e2 = *e1; *e1 = e; *cbest = c; }"),
    "int8_divisor": ("float s = T_E4M3[c] / 127.0f;\n        float z = a / s;",
                     "float s = T_E4M3[c] / 128.0f;\n        float z = a / s;"),
    "sign_dropped": ("int neg = signbit(w[j]) ? 1 : 0;", "int neg = 0;"),
    "tile_h_by_row": ("double c = (mode == ORC_HOPT) ? (double)h[j0 + j] : 1.0;",
                      "double c = (mode == ORC_HOPT) ? (double)h[i0 + i] : 1.0;"),
    "window_short": ("*hi = c0 + window > cmax ? cmax : c0 + window;",
                     "*hi = c0 + window > cmax ? cmax : c0 + window - 1;"),
    "mean_over_r_minus_1": ("(float)(s[j] / (double)rows)", "(float)(s[j] / (double)(rows - 1))"),
    "e2m1_exponent": ("ldexp(1.0 + (double)m / 2.0, e - 1)", "ldexp(1.0 + (double)m / 2.0, e)"),
    "nibble_order": ("if (((j0 + j) & 1) == 0) *p", "if (((j0 + j) & 1) == 1) *p"),
    "e4m3_subnormal": ("v = ldexp((double)m / 8.0, -6);", "v = ldexp((double)m / 8.0, -7);"),
    "ue4m4_bias": ("return ldexp(1.0 + (double)m / 16.0, e - 7);",
                   "return ldexp(1.0 + (double)m / 16.0, e - 8);"),
    "ue5m3_subnormal": ("if (e == 0) return ldexp((double)m / 8.0, -14);",
                        "if (e == 0) return ldexp((double)m / 8.0, -15);"),
    "ue8m0_naive_round_up": ("int c = (ex - 1) - 2 + 127;", "int c = ex - 2 + 127;"),
    "int4_saturates_at_6": ("int q = nearest_rne(T_INT, 8, z);", "int q = nearest_rne(T_INT, 7, z);"),
    "int4_naive_divisor": ("float qmax = (fmt == ORC_NVFP4) ? 6.0f : 7.0f;",
                           "float qmax = (fmt == ORC_NVFP4) ? 6.0f : 6.0f;"),
    "int4_sign_magnitude": (": (uint8_t)((neg ? -q : q) & 15);", ": (uint8_t)((neg << 3) | q);"),
    "ue8m0_skips_code_0": ("case ORC_S_UE8M0: *g = (scale_grid){T_UE8M0, 255, 0}; return 0;",
                           "case ORC_S_UE8M0: *g = (scale_grid){T_UE8M0, 255, 1}; return 0;"),
    "int4_dequant_magnitude": ("int q = (nib & 8) ? 16 - nib : nib;", "int q = nib & 7;"),
    "gram_not_a_mean": ("G[b * B * B + t] = rows > 0 ? (float)(acc[t] / (double)rows) : 0.0f;",
                        "G[b * B * B + t] = rows > 0 ? (float)(acc[t]) : 0.0f;"),
    "gram_wrong_columns": ("acc[i * B + j] += xi * (double)elem(X, dtype, ld, r, b * B + j);",
                           "acc[i * B + j] += xi * (double)elem(X, dtype, ld, r, j);"),
    "gram_diagonal_only": ("            e += (double)Gb[i * B + j] * (d[i] * d[j]);",
                           "            e += (i == j) ? (double)Gb[i * B + j] * (d[i] * d[j]) : 0.0;"),
    "gram_unsigned_difference": ("d[j] = (double)w[j] - (double)copysignf(wq_abs, w[j]);",
                                 "d[j] = (double)fabsf(w[j]) - (double)wq_abs;"),
    "gptq_no_division": ("float err = (wv - wq) / Ub[c * T + c];", "float err = (wv - wq);"),
    "gptq_wrong_sign": ("w[r * T + j] = w[r * T + j] - prod;", "w[r * T + j] = w[r * T + j] + prod;"),
    "gptq_transposed_factor": ("float prod = err * Ub[c * T + j];", "float prod = err * Ub[j * T + c];"),
    "gptq_blocks_no_division": ("err[j] = (wv - wq) / U[p * k + p];", "err[j] = (wv - wq);"),
    "gptq_blocks_wrong_sign": ("w[col[p2]] = w[col[p2]] - acc;", "w[col[p2]] = w[col[p2]] + acc;"),
    "gptq_blocks_transposed_factor": (
        "acc = fmaf(err[j], U[(t * B + j) * k + p2], acc);",
        "acc = fmaf(err[j], U[p2 * k + t * B + j], acc);"),
    "gptq_blocks_no_intrablock": ("w[j0 + j2] = w[j0 + j2] - prod;", "w[j0 + j2] = w[j0 + j2];"),
    "gptq_blocks_search_original": (
        "int c = search_block(fmt, sfmt, mode, window, &g, &w[j0], cw, B, &e1, &e2, &c0);",
        "float w0[256];\n            for (int j = 0; j < B; ++j) w0[j] = elem(W, dtype, ld, i, j0 + j);\n"
        "            int c = search_block(fmt, sfmt, mode, window, &g, w0, cw, B, &e1, &e2, &c0);"),
    "gptq_blocks_perm_ignored": ("int64_t b = perm ? perm[t] : t;", "int64_t b = t;"),
    "gptq_blocks_per_column_subtraction": (
        "for (int j = 0; j < B; ++j) acc = fmaf(err[j], U[(t * B + j) * k + p2], acc);\n"
        "                w[col[p2]] = w[col[p2]] - acc;",
        "for (int j = 0; j < B; ++j) w[col[p2]] = w[col[p2]] - err[j] * U[(t * B + j) * k + p2];"),
    "gptq_blocks_last_residual_only": ("for (int j = 0; j < B; ++j) acc = fmaf(",
                                       "for (int j = B - 1; j < B; ++j) acc = fmaf("),
    "dequant_not_rounded": ("float wq = copysignf(wq_abs, w[j]);\n        double d = (double)w[j] - (double)wq;",
                            "float wq = copysignf(wq_abs, w[j]);\n        double d = (double)w[j] - 1.0000001 * (double)wq;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mut = tmp_path / "oracle_mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-o",
                    str(so), str(mut), "-lm"], check=True)
    env = dict(os.environ, MXQ_ORACLE_LIB=str(so))
    # every pin file runs; the one the mutant's area belongs to first, so that -x stops early
    pins = ["test_oracle_pins.py", "test_oracle_pins_scales.py", "test_oracle_pins_gram.py",
            "test_oracle_pins_gptq.py", "test_oracle_pins_gptq_blocks.py"]
    first = ("test_oracle_pins_gptq_blocks.py" if name.startswith("gptq_blocks") else
             "test_oracle_pins_gptq.py" if name.startswith("gptq") else
             "test_oracle_pins_gram.py" if name.startswith("gram") else
             "test_oracle_pins_scales.py" if name.startswith(("ue", "int4", "mx")) else
             "test_oracle_pins.py")
    pins.remove(first)
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          *[os.path.join(HERE, f) for f in [first] + pins]], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=600)
    assert res.returncode != 0, f"pins did not catch planted mistake {name}:\n{res.stdout[-2000:]}"
