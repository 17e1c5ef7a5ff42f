"""The pins are strong enough: plausible one-line mistakes planted in a copy of
the oracle (compiled separately on the CPU) each fail at least one pin."""
import os
import subprocess

import pytest

import pins
import pins_backward
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


# planted in the backward (reverse-mode) loop; run against the backward pins
BACKWARD_MUTANTS = [
    ("bwd_predict_term_dropped", "for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += kv[i] * dp[j];",
     "for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += 0.0 * dp[j];"),
    ("bwd_dp_sign", "dp[j] = -bv * du[j];", "dp[j] = bv * du[j];"),
    ("bwd_dbeta_without_prediction", "db += du[j] * (vv[j] - pp[j]);", "db += du[j] * vv[j];"),
    ("bwd_dq_unscaled", "dq[tk + i] = c * acc;", "dq[tk + i] = acc;"),
    ("bwd_dq_before_write", "acc += St[(size_t)i * dv + j] * dot[j];", "acc += X[(size_t)i * dv + j] * dot[j];"),
    ("bwd_dlog_alpha_undecayed", "acc += G[(size_t)i * dv + j] * X[(size_t)i * dv + j];",
     "acc += G[(size_t)i * dv + j] * Sp[(size_t)i * dv + j];"),
    ("bwd_cotangent_not_decayed", "for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] *= ai;",
     "for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] *= 1.0;"),
    ("bwd_wrong_checkpoint", "memcpy(cur, ckpt + DD * (size_t)n, sizeof(double) * DD);",
     "memcpy(cur, ckpt + DD * (size_t)(n > 0 ? n - 1 : 0), sizeof(double) * DD);"),
    ("bwd_dk_write_term_dropped", "acc += G[(size_t)i * dv + j] * uu[j];", "acc += 0.0 * uu[j];"),
]


def _build_mutant(tmp_path, name, orig, bad):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"mutation anchor for {name} not found exactly once"
    mutant_c = tmp_path / f"mutant_{name}.c"
    mutant_c.write_text(src.replace(orig, bad))
    so = tmp_path / f"libmutant_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                           "-o", str(so), str(mutant_c), "-lm"])
    return orc.load_library(str(so))


@pytest.mark.parametrize("name,orig,bad", BACKWARD_MUTANTS, ids=[m[0] for m in BACKWARD_MUTANTS])
def test_backward_mutant_is_caught(tmp_path, name, orig, bad):
    lib = _build_mutant(tmp_path, name, orig, bad)
    failed = []
    for check in pins_backward.BACKWARD_CHECKS:
        try:
            check(lib=lib)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no backward pin catches the planted mistake {name}"


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
