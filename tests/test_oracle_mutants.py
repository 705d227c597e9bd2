"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of oracle.c (on the CPU, in a temporary
directory), builds it, and runs the pin tests against that build; at least one
pin must fail.  A mutant that survives would mean the pins leave that part of
the oracle unchecked.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "zero_sign": ("float z32 = rintf(-mn / sf);", "float z32 = rintf(mn / sf);"),
    "floor_not_rint": ("float qf = rintf(t) + zf;", "float qf = floorf(t) + zf;"),
    "codes_ties_away": ("float qf = rintf(t) + zf;", "float qf = roundf(t) + zf;"),
    "zero_ties_away": ("float z32 = rintf(-mn / sf);", "float z32 = roundf(-mn / sf);"),
    "scale_denominator": ("float s32 = r / Q;", "float s32 = r / (Q + 1.0f);"),
    "group_row_index": ("const uint16_t* w = W + row * k + g * group;", "const uint16_t* w = W + g * group;"),
    "pack_low_first": ("byte |= (q & ((1u << bits) - 1)) << (8 - bits * (t + 1));",
                       "byte |= (q & ((1u << bits) - 1)) << (bits * t);"),
    "dequant_plus_zero": ("float d = (float)q - zf;", "float d = (float)q + zf;"),
    "codebook_tie_upper": ("if (d < bestd) { bestd = d; best = j; }", "if (d <= bestd) { bestd = d; best = j; }"),
    "codebook_unnormalised": ("float x = (a == 0.0f) ? 0.0f : oracle_bf16_to_f32(w[i]) / a;",
                              "float x = (a == 0.0f) ? 0.0f : oracle_bf16_to_f32(w[i]);"),
    "absmax_halved": ("if (v > a) a = v;", "if (v > a) a = v * 0.5f;"),
    "dq_128_levels": ("float u = t * 127.0f;", "float u = t * 128.0f;"),
    "dq_offset_count": ("float off = (float)(sum / (double)nb);", "float off = (float)(sum / (double)(nb + 1));"),
    "fwd_lora_sign": ("if (Y) Y[i * n + j] = acc + s * lora;", "if (Y) Y[i * n + j] = acc - s * lora;"),
    "fwd_B_transposed": ("double b = oracle_bf16_to_f32(B[j * r + u]);\n                lora += t[u] * b;",
                         "double b = oracle_bf16_to_f32(B[u * n + j]);\n                lora += t[u] * b;"),
    "bwd_dropped_scale": ("if (dX) dX[i * k + c] = acc + s * lora;", "if (dX) dX[i * k + c] = acc + lora;"),
    "bwd_W_not_transposed": ("double w = W_hat[j * k + c];\n                acc += g * w;",
                             "double w = W_hat[(c % n) * k + j % k];\n                acc += g * w;"),
    "dA_uses_T": ("acc += U[i * r + t] * x;", "acc += T[i * r + t] * x;"),
    "dB_missing_s": ("if (dB) dB[j * r + t] = s * acc;", "if (dB) dB[j * r + t] = acc;"),
    "merge_missing_s": ("float t = s * d;", "float t = d;"),
    "merge_sign_ignored": ("float v = (sign > 0) ? W_in[row * k + col] + t : W_in[row * k + col] - t;",
                           "float v = W_in[row * k + col] + t;"),
    "merge_A_transposed": ("oracle_bf16_to_f32(A[(int64_t)u * k + col])", "oracle_bf16_to_f32(A[col * r + u])"),
    "merge_truncates": ("if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u;", "(void)lo;"),
    "merge_ties_away": ("if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u;", "if (lo >= 0x8000u) hi += 1u;"),
    "score_sign": ("sc += m2[j] * (e2 * e2 - e4 * e4);", "sc += m2[j] * (e4 * e4 - e2 * e2);"),
    "score_first_moment": ("acc += x * x;", "acc += x;"),
    "select_ties_upper": ("(score[d] == score[c] && d < c)", "(score[d] == score[c] && d > c)"),
    "merge_reordered_sum": ("for (int u = 0; u < r; ++u)\n                d = fmaf(", "for (int u = r - 1; u >= 0; --u)\n                d = fmaf("),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new)
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "oracle.c")
        open(c, "w").write(mutated)
        open(os.path.join(d, "oracle.h"), "w").write(open(os.path.join(ROOT, "oracle", "oracle.h")).read())
        so = os.path.join(d, "liboracle_mut.so")
        subprocess.check_call(["gcc", "-std=c11", "-O1", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                               "-w", "-o", so, c, "-lm"])
        env = dict(os.environ, LBQ_ORACLE_LIB=so, OMP_NUM_THREADS="2")
        res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                              os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                             cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        assert res.returncode != 0, f"mutant {name} survived the pins:\n{res.stdout[-2000:]}"
