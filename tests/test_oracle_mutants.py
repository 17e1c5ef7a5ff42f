"""The pins are strong enough: plausible one-line mistakes planted in a copy of
the oracle (compiled separately on the CPU) each fail at least one pin."""
import os
import subprocess

import pytest

import pins
from oracle import oracle as orc

SRC = os.path.join(os.path.dirname(orc.__file__), "kda_oracle.c")

# (name, original line fragment, planted mistake)
MUTANTS = [
    ("error_sign", "u[j] = bt * (vt[j] - p[j]);", "u[j] = bt * (vt[j] + p[j]);"),
    ("beta_dropped", "u[j] = bt * (vt[j] - p[j]);", "u[j] = (vt[j] - p[j]);"),
    ("beta_squared", "u[j] = bt * (vt[j] - p[j]);", "u[j] = bt * bt * (vt[j] - p[j]);"),
    ("decay_growth", "const double a = exp(lat[i]);", "const double a = exp(-lat[i]);"),
    ("scalar_decay", "const double a = exp(lat[i]);", "const double a = exp(lat[0]);"),
    ("predict_with_query", "p[j] += S[(size_t)i * dv + j] * kt[i];",
     "p[j] += S[(size_t)i * dv + j] * qt[i];"),
    ("write_with_query", "S[(size_t)i * dv + j] += kt[i] * u[j];",
     "S[(size_t)i * dv + j] += qt[i] * u[j];"),
    ("read_before_write", "ot[j] += S[(size_t)i * dv + j] * qt[i];",
     "ot[j] += (S[(size_t)i * dv + j] - kt[i] * u[j]) * qt[i];"),
    ("scale_1_over_dk", "1.0 / sqrt((double)dk)", "1.0 / (double)dk"),
    ("first_channel_never_decays", "for (int i = 0; i < dk; ++i) {\n                const double a",
     "for (int i = 1; i < dk; ++i) {\n                const double a"),
]


@pytest.mark.parametrize("name,orig,bad", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, orig, bad):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"mutation anchor for {name} not found exactly once"
    mutant_c = tmp_path / f"mutant_{name}.c"
    mutant_c.write_text(src.replace(orig, bad))
    so = tmp_path / f"libmutant_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                           "-o", str(so), str(mutant_c), "-lm"])
    lib = orc.load_library(str(so))
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check(lib=lib)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no pin catches the planted mistake {name}"
