"""The oracle pins must fail for plausible mistakes in the oracle (mutation test, CPU only).

Each case copies msa_oracle.c, applies one textual mutation (a dropped term, a wrong sign,
index or divisor, a swapped operand), compiles the copy and runs the pin suite against it
through MSA_ORACLE_LIB. The pin suite must fail for every mutant.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "msa_oracle.c")

MUTANTS = {
    "pool_divisor": ("pooled[(g * nb_cap + j) * dI + i] = sum / (double)Bk;",
                     "pooled[(g * nb_cap + j) * dI + i] = sum / (double)(Bk + 1);"),
    "pool_transposed_index": ("sum += oracle_bf16_to_f64(k_idx[(t * G + g) * dI + i]);\n                pooled",
                              "sum += oracle_bf16_to_f64(k_idx[(g * N + t) * dI + i]);\n                pooled"),
    "score_scale_dropped": ("s[j] = dot * scale;", "s[j] = dot;"),
    "tie_break_reversed": ("(sa == sb && ja < jb)", "(sa == sb && ja > jb)"),
    "one_block_too_few": ("for (int64_t r = 0; r < topk - 1; ++r) {\n            int64_t best",
                          "for (int64_t r = 0; r < topk - 2; ++r) {\n            int64_t best"),
    "diagonal_dropped": ("        free(taken);\n        sel[n++] = (int32_t)c;", "        free(taken);"),
    "softmax_scale": ("    double scale = 1.0 / sqrt((double)d);", "    double scale = 1.0 / sqrt((double)d * 2.0);"),
    "causal_self_excluded": ("use[u] = (sel == NULL) || block_selected(u / Bk, sel, nsel);\n        if (!use[u]) continue;\n"
                             "        double dot = 0.0;\n        for (int64_t i = 0; i < d; ++i) dot += qd[i] * oracle_bf16_to_f64(K[u * d + i]);\n"
                             "        z[u] = dot * scale;",
                             "use[u] = (u < t || t == 0) && ((sel == NULL) || block_selected(u / Bk, sel, nsel));\n        if (!use[u]) continue;\n"
                             "        double dot = 0.0;\n        for (int64_t i = 0; i < d; ++i) dot += qd[i] * oracle_bf16_to_f64(K[u * d + i]);\n"
                             "        z[u] = dot * scale;"),
    "pv_uses_keys": ("o[i] += p * oracle_bf16_to_f64(V[u * d + i]);", "o[i] += p * oracle_bf16_to_f64(K[u * d + i]);"),
    "topk_ties_to_higher_column": ("    return ja < jb;\n}\n\n/* idx[row][r]", "    return ja > jb;\n}\n\n/* idx[row][r]"),
    "topk_nan_ranked_low": ("    if (na != nb) return na;", "    if (na != nb) return nb;"),
    "topk_ascending": ("    if (!na && a != b) return a > b;", "    if (!na && a != b) return a < b;"),
    "e4m3_bias": ("    else v = ldexp(1.0 + m / 8.0, e - 7);", "    else v = ldexp(1.0 + m / 8.0, e - 8);"),
    "e4m3_ties_to_odd": ("if (dist < bd || (dist == bd && (c & 1) == 0))", "if (dist < bd || (dist == bd && (c & 1) == 1))"),
    "fp8_scale_divisor": ("amax > 0.0f ? amax / 448.0f : 1.0f", "amax > 0.0f ? amax / 240.0f : 1.0f"),
    "fp8_open_block_from_codes": ("            const double k = j < c ?", "            const double k = j <= c ?"),
    "grad_dz_sign": ("const double dz = p[u] * (dp - dOo);", "const double dz = p[u] * (dp + dOo);"),
    "grad_dq_unscaled": ("dQ[i] += s * dz * oracle_bf16_to_f64(K[u * d + i]);", "dQ[i] += dz * oracle_bf16_to_f64(K[u * d + i]);"),
    "grad_dk_uses_keys": ("dK[u * d + i] += s * dz * qd[i];", "dK[u * d + i] += s * dz * oracle_bf16_to_f64(K[u * d + i]);"),
    "score_sign": ("dot += oracle_bf16_to_f64(q_idx_row[i]) * pooled_g[j * dI + i];",
                   "dot -= oracle_bf16_to_f64(q_idx_row[i]) * pooled_g[j * dI + i];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} must occur exactly once"
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", str(mut),
                           "-o", str(so), "-lm"])
    env = dict(os.environ, MSA_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
