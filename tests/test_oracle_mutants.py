"""Each plausible mistake planted in a copy of the oracle fails a pin.

Every mutant below is a one-line edit of ``oracle/oracle.c`` (a flipped sign,
a wrong index, a dropped term, a transposed operand, a swapped operand).  The
copy is compiled to a temporary library on the CPU and the pin suite
(tests/test_oracle_pins.py) is run against it in a subprocess; the suite must
fail.  All mutants stay in bounds: none reads outside its arrays.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "rope_sign": ("y[i] = x0 * c - x1 * s;", "y[i] = x0 * c + x1 * s;"),
    "rope_theta": ("pow(base, -2.0 * (double)i / (double)d)", "pow(base, -1.0 * (double)i / (double)d)"),
    "rope_pairing": ("double x0 = x[i], x1 = x[i + half];", "double x0 = x[i], x1 = x[half - 1 - i];"),
    "head_to_unit": ("const int32_t h = u * G + g;", "const int32_t h = g * U + u;"),
    "tie_break": ("if (x->t < y->t) return -1;\n  if (x->t > y->t) return 1;",
                  "if (x->t > y->t) return -1;\n  if (x->t < y->t) return 1;"),
    "group_sum_dropped": ("s_u[t] += acc;", "s_u[t] = acc;"),
    "qlat_unit_rows": ("acc += qh[i] * Pk_u[(int64_t)i * r + c];", "acc += qh[i] * C->Pk[(int64_t)i * r + c];"),
    "reconstruct_transposed": ("ak += kc[c] * Pk_u[(int64_t)i * r + c];", "ak += kc[c] * Pk_u[(int64_t)c * d + i];"),
    "pv_pk_swapped": ("av += vc[c] * Pv_u[(int64_t)i * r + c];", "av += vc[c] * Pk_u[(int64_t)i * r + c];"),
    "scale_dropped": ("logit[j] = acc * scale;", "logit[j] = acc;"),
    "key_position": ("oracle_rope(Ksel + j * d, d, (double)sel[j],", "oracle_rope(Ksel + j * d, d, (double)(sel[j] + 1),"),
    "query_position": (": (double)nb;", ": (double)(nb - 1);"),
    "softmax_unnormalised": ("double p = logit[j] / den;", "double p = logit[j];"),
    "sequence_offset": ("const double* Kc_b = C->Kc + off * r;", "const double* Kc_b = C->Kc;"),
    "compress_transposed": ("acc += x[h] * j->P[(int64_t)h * j->r + c];", "acc += x[h] * j->P[(int64_t)c * j->hid + h];"),
    "bf16_ties_away": ("double y = ldexp(nearbyint(ldexp(m, 8)), e - 8);", "double y = ldexp(round(ldexp(m, 8)), e - 8);"),
    "threshold_strict": ("!(order[j].s >= D->select_threshold)", "!(order[j].s > D->select_threshold)"),
    "bf16_width": ("double y = ldexp(nearbyint(ldexp(m, 8)), e - 8);", "double y = ldexp(nearbyint(ldexp(m, 9)), e - 9);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new)
    c_path = tmp_path / "oracle_mutant.c"
    so_path = tmp_path / "liboracle_mutant.so"
    c_path.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                    "-o", str(so_path), str(c_path), "-lm"], check=True)
    env = dict(os.environ, SALS_ORACLE_LIB=str(so_path))
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode != 0, f"mutant {name} passed every pin:\n{res.stdout[-2000:]}"
