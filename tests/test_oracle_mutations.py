"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a temporary copy of ``oracle/spark_oracle.c``
(a dropped term, a wrong sign, a wrong index, a wrong reading of std), builds
it with gcc, and runs ``tests/test_oracle_pins.py`` against it in a
subprocess.  The pin suite must fail for every planted mistake.  CPU only; the
committed oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "spark_oracle.c")

MUTATIONS = {
    "sample_std": ("sqrt(ss / (double)d)", "sqrt(ss / (double)(d - 1))"),
    "theta_sign": ("return mean + sd * oracle_topk_quantile", "return mean - sd * oracle_topk_quantile"),
    "variance_drops_mean": ("double c = x[i] - mean;", "double c = x[i];"),
    "gelu_cubic_term": ("0.044715 * s * s * s", "0.044715 * s * s"),
    "bisection_direction": ("lo = mid; /* too much", "hi = mid; /* too much"),
    "a_uses_q_head": ("* oracle_bf16_to_f64(qt[r + j])", "* oracle_bf16_to_f64(qt[j])"),
    "K1_transposed": ("K1[i * r + j]", "K1[j * r + i]"),
    "V_wrong_row": ("V[i * d_model + c]", "V[(d_ff - 1 - i) * d_model + c]"),
    "gelu_of_x_not_s": ("double g = gelu_of_kind(s, gelu_kind);", "double g = gelu_of_kind(x[i], gelu_kind);"),
    "drops_a": ("double h = g * a;", "double h = g;"),
    "soft_threshold_not_clamped": ("out[row * d + i] = s > 0.0 ? s : 0.0;", "out[row * d + i] = s;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fopenmp",
                           "-fPIC", "-shared", str(mutated), "-o", str(lib), "-lm"])
    env = dict(os.environ, SPARK_ORACLE_LIB=str(lib))
    proc = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                          env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert proc.returncode != 0, f"pins did not catch mutation {name}:\n{proc.stdout[-2000:]}"
