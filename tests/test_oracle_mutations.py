"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a private copy of the oracle's C source (on the
CPU, in a temporary directory), builds it, and runs the pin suite against that
build; the suite must fail. The committed oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lsh_oracle.c")

# (name, text in the oracle, planted replacement)
MUTANTS = [
    ("keys-not-normalised", "l = (nrm > 0.0) ? dot / nrm * inv_sqrt_d : 0.0;",
     "l = dot * inv_sqrt_d;"),
    ("no-sqrt-d-scale", "l = (nrm > 0.0) ? dot / nrm * inv_sqrt_d : 0.0;",
     "l = (nrm > 0.0) ? dot / nrm : 0.0;"),
    ("self-not-masked", "if (pj == ps) {", "if (0) {"),
    ("next-chunk-not-previous", "const int lo = (c > 0 ? c - 1 : 0) * mc;\n        const int hi = (c + 1) * mc;",
     "const int lo = c * mc;\n        const int hi = (c + 2) * mc > n ? n : (c + 2) * mc;"),
    ("own-chunk-only", "const int lo = (c > 0 ? c - 1 : 0) * mc;", "const int lo = c * mc;"),
    ("causal-reversed", "if (causal && pj > ps) continue;", "if (causal && pj < ps) continue;"),
    ("hash-halves-swapped", "c[j] = p[j];\n            c[half + j] = -p[j];",
     "c[j] = -p[j];\n            c[half + j] = p[j];"),
    ("hash-last-index-tie", "if (c[t] > c[best]) best = t;", "if (c[t] >= c[best]) best = t;"),
    ("hash-R-transposed", "for (int j = 0; j < half; ++j) p[j] += xk * Rk[j];",
     "for (int j = 0; j < half; ++j) p[j] += xk * R[((int64_t)j * d + k) % ((int64_t)d * half)];"),
    ("sort-unstable", "for (int i = 0; i < n; ++i) {\n        const int64_t s = start[bucket[i]]++;",
     "for (int i = n - 1; i >= 0; --i) {\n        const int64_t s = start[bucket[i]]++;"),
    ("merge-uniform-weights", "const double w = exp(lse[r * npos + i] - lsum);",
     "const double w = 1.0 / rounds;"),
    ("self-logit-added", "l = LSHO_SELF_LOGIT;",
     "l = LSHO_SELF_LOGIT + 1.0;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                    "-o", str(lib), str(mutant), "-lm"], check=True)
    env = dict(os.environ, LSH_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
