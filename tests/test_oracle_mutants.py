"""Planted mistakes in the oracle: each is a plausible slip in its arithmetic, and each must
make at least one pin fail (the CPU tests of tests/test_oracle_pins.py and
tests/test_golden.py).

Every mutant is a copy of oracle/dr_oracle.c with one textual change, compiled with gcc into
a temporary directory. The pins then run in a subprocess whose `oracle` fixture loads that
library. Nothing here touches the GPU or the product path.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dr_oracle.c")

RESID = "const double r = vv[i] - pred[i];"
WRITE = "S[ij] = decay[j] * S[ij] + b * r * kk[j];"
DECAY = "if (!residual_pre_decay) s *= decay[j];"
UOUT = "if (ut) ut[i] = b * r;"
MUTANTS = {
    "residual_sign": [(RESID, "const double r = vv[i] + pred[i];")],
    "dropped_prediction": [(RESID, "const double r = vv[i];")],
    "beta_on_v_not_write": [(RESID, "const double r = b * vv[i] - pred[i];"),
                            (WRITE, "S[ij] = decay[j] * S[ij] + r * kk[j];")],
    "kda_decay_on_rows": [(DECAY, "if (!residual_pre_decay) s *= decay[i % dk];"),
                          (WRITE, "S[ij] = decay[i % dk] * S[ij] + b * r * kk[j];")],
    "gdn2_writes_along_k": [(WRITE, "S[ij] = decay[j] * S[ij] + b * r * kt[j];")],
    "gdn2_reads_along_k": [("acc += s * kk[j];", "acc += s * kt[j];")],
    "gdn2_target_ignores_write_gate": [("z[i] = write[t * dv + i] * vt[i];", "z[i] = vt[i];")],
    "gdn2_erase_ignores_gate": [("e[j] = erase[t * dk + j] * kt[j];", "e[j] = kt[j];")],
    "gdn2_without_decay": [("else if (mode == ORACLE_GDN || mode == ORACLE_GDN2) decay[j] = gate[t];",
                            "else if (mode == ORACLE_GDN) decay[j] = gate[t];\n"
                            "                else if (mode == ORACLE_GDN2) decay[j] = 1.0;")],
    "write_value_without_beta": [(UOUT, "if (ut) ut[i] = r;")],
    "write_value_is_the_target": [(UOUT, "if (ut) ut[i] = b * vv[i];")],
    "residual_against_undecayed_state": [(DECAY, "if (0) s *= decay[j];")],
    "readout_of_transposed_state": [
        ("for (int j = 0; j < dk; ++j) acc += S[(long)i * dk + j] * qt[j];",
         "for (int j = 0; j < dk; ++j) acc += S[(long)(j % dv) * dk + (i % dk)] * qt[j];")],
    "sherman_morrison_without_u_z": [("for (int i = 0; i < d; ++i) den += ut[i] * z[i];",
                                      "for (int i = 0; i < d; ++i) den += 0.0 * ut[i] * z[i];")],
    "vla_direction_not_normalised": [("const double inv = 1.0 / sqrt(nrm2);",
                                      "const double inv = 1.0;")],
    "vla_writes_along_k": [("S[(long)i * d + j] += r[i] * y[j];",
                            "S[(long)i * d + j] += r[i] * kt[j];")],
    "vla_ratio_normalizer_along_k": [("for (int j = 0; j < d; ++j) n[j] += (1.0 - nk) * y[j];",
                                      "for (int j = 0; j < d; ++j) n[j] += (1.0 - nk) * kt[j];")],
    "vla_ratio_normalizer_accumulates": [
        ("for (int j = 0; j < d; ++j) n[j] += (1.0 - nk) * y[j];",
         "for (int j = 0; j < d; ++j) n[j] += y[j];")],
    "vla_ratio_without_division": [("ot[i] = n ? acc / nq : acc;", "ot[i] = acc;")],
    "loglinear_merge_drops_lower_levels": [("for (int b = 0; b < jt; ++b) x += M[b * state + e];",
                                            "for (int b = 0; b < 0; ++b) x += M[b * state + e];")],
    "loglinear_level_weights_shifted": [("acc += lt[b + 1] * lev;", "acc += lt[b] * lev;")],
    "loglinear_counter_on_trailing_zeros": [("while ((t >> jt) & 1) ++jt;",
                                             "while (jt < 30 && !((t >> jt) & 1)) ++jt;")],
    "loglinear_without_own_token": [("acc *= lt[0];", "acc *= 0.0;")],
}


def run_pins(tmp_path, src: str):
    """Compile `src` as the oracle library and run the pins against it; returns the run."""
    csrc = tmp_path / "mutant.c"
    csrc.write_text(src)
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(lib), str(csrc),
                           "-lm"])
    env = dict(os.environ, ORACLE_MUTANT_LIB=str(lib))
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           "-m", "not gpu", "tests/test_oracle_pins.py", "tests/test_golden.py"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_unmodified_oracle_passes_the_pins_by_the_same_route(tmp_path):
    run = run_pins(tmp_path, open(SRC).read())
    assert run.returncode == 0, run.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_fails_a_pin(tmp_path, name):
    src = open(SRC).read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, (name, old)  # the mutation still targets real code
        src = src.replace(old, new)
    run = run_pins(tmp_path, src)
    assert run.returncode == 1, (name, run.stdout[-2000:])  # 1 = tests ran and some failed
