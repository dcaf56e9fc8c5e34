"""The oracle's pins catch plausible mistakes (CPU only).

Each case copies oracle.c, plants one mistake (a dropped or sign-flipped term,
a wrong index, a transposed operand, a wrong rounding rule, a wrong bit order),
builds the copy, and runs the pin suite against it: the suite must fail.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "residual_sign": ("v = v + oracle_f16_to_f64(*e2);", "v = v - oracle_f16_to_f64(*e2);"),
    "residual_dropped_exact": ("  if (h2) {\n    int s2, e2;", "  if (0) {\n    int s2, e2;"),
    "ties_away": ("if (rem > half || (rem == half && (N & 1))) N += 1;", "if (rem >= half) N += 1;"),
    "msb_first": ("uint32_t b = (row[bit >> 3] >> (bit & 7)) & 1u;", "uint32_t b = (row[bit >> 3] >> (7 - (bit & 7))) & 1u;"),
    "element_reversed": ("*h1 = main_entry(L, g, i1, q % d);", "*h1 = main_entry(L, g, i1, d - 1 - q % d);"),
    "replace_dropped": ("W[(int64_t)i * ldw + L->col_idx[e]] = L->values[e];   /* REPLACE: exact outliers */", ";"),
    "operand_reversed": ("for (int32_t j = 0; j < L->n_in; ++j) acc += w[j] * x[j];",
                         "for (int32_t j = 0; j < L->n_in; ++j) acc += w[j] * x[L->n_in - 1 - j];"),
    "subnormal_exponent": ("if (e == 0) { *mant = f; *exp2 = -24; }", "if (e == 0) { *mant = f; *exp2 = -25; }"),
    "outlier_codebook": ("*h1 = *(L->cbo + (int64_t)io * d + (p % d));",
                         "*h1 = *(L->cb1 + (int64_t)(io % L->k1) * d + (p % d));"),
    "col_scale_dropped": ("if (L->cs) v = v * oracle_f16_to_f64(L->cs[j]);", ";"),
    "assign_ties_highest": ("if (i == 0 || D < best_d) {", "if (i == 0 || D <= best_d) {"),
    "assign_residual_dropped": ("      for (int32_t t = 0; t < d; ++t) v[t] -= f16_units(C1[(int64_t)i1 * d + t]);\n",
                                "\n"),
    "assign_element_skewed": ("i128 diff = (i128)v[t] - (i128)f16_units(c[t]);",
                              "i128 diff = (i128)v[t] - (i128)f16_units(c[(t + 1) % d]);"),
    "assign_sum_not_difference": ("i128 diff = (i128)v[t] - (i128)f16_units(c[t]);",
                                  "i128 diff = (i128)v[t] + (i128)f16_units(c[t]);"),
    "group_offset_dropped": ("if (!L->cb_symmetry) return L->cb1[((int64_t)g * L->k1 + i1) * d + e];",
                             "if (!L->cb_symmetry) return L->cb1[((int64_t)0 * L->k1 + i1) * d + e];"),
    "group_size_floor": ("  const int32_t size = (n_sub + G - 1) / G;", "  const int32_t size = n_sub / G > 0 ? n_sub / G : 1;"),
    "sym_patterns_swapped": ("(t == 2 && (e & 1)) || (t == 3 && !(e & 1))", "(t == 3 && (e & 1)) || (t == 2 && !(e & 1))"),
    "vsr_dropped": ("if (q < n_main_cols(L)) W[(int64_t)i * ldw + main_col[q]] = L->vsr_values[(int64_t)b * L->d + t];",
                    ";"),
    "vsr_element_shift": ("          const int32_t q = L->vsr_pos[b] * L->d + t;\n",
                          "          const int32_t q = L->vsr_pos[b] * L->d + (t + 1) % L->d;\n"),
    "assign_units_truncated": ("  int64_t v = m << (e + 24);", "  int64_t v = (m << (e + 24)) >> 4 << 4;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_fail_on_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation site not found: " + name
    mutant_c = tmp_path / "oracle_mutant.c"
    mutant_c.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=gnu99", "-ffp-contract=off", "-fPIC", "-shared",
                           str(mutant_c), "-o", str(lib), "-lm"])
    env = dict(os.environ, VQ_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "pins did not notice mutant %s:\n%s" % (name, r.stdout[-2000:])
