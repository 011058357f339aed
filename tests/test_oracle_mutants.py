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


def _run_mutant(tmp, name, old, new):
    src = open(SRC).read()
    if src.count(old) != 1:
        return None, f"mutation anchor for {name} not found once"
    d = os.path.join(tmp, name)
    os.makedirs(d)
    mut = os.path.join(d, "oracle_mut.c")
    with open(mut, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(d, "liboracle_mut.so")
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", mut, "-o", so, "-lm"],
                   check=True)
    env = dict(os.environ, ORACLE_LIB_OVERRIDE=so, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_runs(tmp_path_factory):
    """Every mutant's pin run, the runs side by side (one process each)."""
    import concurrent.futures as cf
    tmp = str(tmp_path_factory.mktemp("mutants"))
    with cf.ThreadPoolExecutor(max_workers=min(len(MUTANTS), os.cpu_count() or 1)) as ex:
        futs = {m[0]: ex.submit(_run_mutant, tmp, *m) for m in MUTANTS}
        return {k: f.result() for k, f in futs.items()}


@pytest.mark.slow
@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_pins_catch_mutant(mutant_runs, name):
    rc, out = mutant_runs[name]
    assert rc is not None, out
    assert rc != 0, f"pins did not catch mutant {name}:\n{out}"
