"""The oracle's pins must catch plausible mistakes in the oracle itself.

Each case below plants one mistake in a copy of oracle/oracle.c (on the CPU,
in a temporary directory), builds it, and runs the pin suite against that
build; the suite must fail.  The unmodified source must pass (checked by
tests/test_oracle_pins.py itself).
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = [
    ("dropped_scale", "z[j] = scale * s;", "z[j] = s;"),
    ("flipped_shift_sign", "double p = exp(z[j] - m);", "double p = exp(m - z[j]);"),
    ("scores_use_values", "for (int e = 0; e < d; ++e) s += q[e] * k[j * stride + e];",
     "for (int e = 0; e < d; ++e) s += q[e] * v[j * stride + e];"),
    ("prefill_not_causal", "v + (int64_t)h * d, i + 1, stride,", "v + (int64_t)h * d, P, stride,"),
    ("ring_never_advances", "r->ring_pos = (r->ring_pos + 1) % r->window;",
     "r->ring_pos = r->ring_pos % r->window;"),
    ("warmup_one_short", "if (r->len < r->prefill_len + r->window) {",
     "if (r->len < r->prefill_len + r->window - 1) {"),
    ("ngram_prefix_shifted", "const int32_t *prefix = hist + (h - n + 1);",
     "const int32_t *prefix = hist + (h - n);"),
    ("ngram_last_start_dropped", "for (int i = 0; i + n <= h; ++i) {", "for (int i = 0; i + n < h; ++i) {"),
    ("ngram_no_vocab_check", "if (hist[i] < 0 || hist[i] >= vocab) ok = 0;", "ok = ok;"),
]


@pytest.mark.slow
@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found once"
    mut = tmp_path / "oracle_mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mut.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", str(mut), "-o", str(so),
                    "-lm"], check=True)
    env = dict(os.environ, ORACLE_LIB_OVERRIDE=str(so), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
