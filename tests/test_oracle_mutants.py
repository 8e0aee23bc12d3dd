"""Plants plausible mistakes in a temporary copy of the fp64 oracle (CPU only)
and checks that the pins in test_oracle_pins.py reject every one of them.

The committed oracle is never modified: each mutant is a string edit of a copy
of kd_oracle.c compiled into a temporary directory and loaded through a copy
of oracle.py.
"""
import importlib.util
import os
import shutil

import pytest

import tests.test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "kd_oracle.c")
PY = os.path.join(ROOT, "oracle", "oracle.py")

# (name, exact text in kd_oracle.c, replacement)
MUTANTS = [
    ("erase-sign", "double u = c - beta * b;", "double u = c + beta * b;"),
    ("no-decay", "S[(size_t)r * dk + j] *= exp(logf[j]);", "S[(size_t)r * dk + j] *= 1.0;"),
    ("decay-on-rows", "S[(size_t)r * dk + j] *= exp(logf[j]);",
     "S[(size_t)r * dk + j] *= exp(logf[r % dk]);"),
    ("write-transposed", "S[(size_t)r * dk + j] += u * v[r] * k[j];",
     "S[(size_t)r * dk + j] += u * v[j % dv] * k[r % dk];"),
    ("read-with-k", "acc += S[(size_t)r * dk + j] * q[j];", "acc += S[(size_t)r * dk + j] * k[j];"),
    ("assoc-uses-q", "row += S[(size_t)r * dk + j] * k[j];", "row += S[(size_t)r * dk + j] * q[j];"),
    ("bwd-dbeta-sign", "jb->dbeta[g] = -bb * du;", "jb->dbeta[g] = bb * du;"),
    ("bwd-dq-prev-state", "acc += Scur[(size_t)r * DK + j] * dOt[r];",
     "acc += Sprev[(size_t)r * DK + j] * dOt[r];"),
    ("bwd-no-state-decay", "G[(size_t)r * DK + j] *= exp(lf[j]);", "G[(size_t)r * DK + j] *= 1.0;"),
    ("bwd-dlogf-before-erase", "accl += G[(size_t)r * DK + j] * Sbar[(size_t)r * DK + j];",
     "accl += (G[(size_t)r * DK + j] - db * vt[r] * kt[j]) * Sbar[(size_t)r * DK + j];"),
    ("bwd-dv-missing-erase-term", "dvt[r] += db * acc;", "dvt[r] += 0.0 * acc;"),
]

PIN_TESTS = [
    lambda o: pins.test_write_hits_target(o, "general"),
    lambda o: pins.test_interference_formula_and_orthogonal_protection(o),
    lambda o: pins.test_non_expansive(o, 2.0),
    lambda o: pins.test_bruteforce_vectorised_products(o, 4, 3, 12),
    lambda o: pins.test_beta_zero_gated_linear_attention(o),
    lambda o: pins.test_dv1_reduces_to_kda(o),
    lambda o: pins.test_reverse_recurrence_finite_differences(o, 64),
]


def _load_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    d = tmp_path / name
    d.mkdir()
    (d / "kd_oracle.c").write_text(src.replace(old, new))
    shutil.copy(PY, d / "oracle.py")
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{name.replace('-', '_')}", d / "oracle.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build_oracle(force=True)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_every_mutant_fails_a_pin(tmp_path, name, old, new):
    mod = _load_mutant(tmp_path, name, old, new)
    caught = False
    for pin in PIN_TESTS:
        try:
            pin(mod)
        except AssertionError:
            caught = True
            break
    assert caught, f"mutant {name} passed every pin"
