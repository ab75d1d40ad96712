"""Plant plausible mistakes in a copy of the oracle and check that the pins fail.

Each mutation is a one-line edit of ``oracle/efla_oracle.c`` compiled into a
temporary library; the pin suite is then run against it in a subprocess
(``EFLA_ORACLE_SO`` points the oracle loader at the mutant) and must fail.
The mistakes planted are the ones a reader of the pages could make: a
dropped write term, lambda = ||k|| instead of ||k||^2, the sign of expm1 as
printed in one blog, 1 - exp instead of expm1, a missing epsilon clamp, a
transposed readout S q, and a chunked output that drops the diagonal of
tril(Q K^T).
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "efla_oracle.c")

MUTATIONS = {
    "dropped_write_term": ("+= -a * k[i] * kts[j] + a * k[i] * v[j];", "+= -a * k[i] * kts[j];"),
    "lambda_is_norm": ("double a = efla_oracle_alpha(beta[row], lam, euler);",
                       "double a = efla_oracle_alpha(beta[row], sqrt(lam), euler);"),
    "expm1_sign": ("return -expm1(-beta * lc) / lc;", "return expm1(-beta * lc) / lc;"),
    "one_minus_exp": ("return -expm1(-beta * lc) / lc;", "return (1.0 - exp(-beta * lc)) / lc;"),
    "no_clamp": ("double lc = lambda > EFLA_ORACLE_EPS ? lambda : EFLA_ORACLE_EPS;",
                 "double lc = lambda;"),
    "transposed_readout": ("o[j] += S[(long)i * dv + j] * q[i];",
                           "o[j] += S[(long)j * dv + i] * q[i];"),
    "chunk_tril_strict": ("for (int m = 0; m <= r; ++m) {\n                        double qk",
                          "for (int m = 0; m < r; ++m) {\n                        double qk"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", str(so),
                    str(mut), "-lm"], check=True)
    env = dict(os.environ, EFLA_ORACLE_SO=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not notice mutation {name}:\n{r.stdout[-2000:]}"
