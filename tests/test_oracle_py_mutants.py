"""The pins of the oracle's numpy functions (selection, sampling, RoPE, the
banded prefill, the partial/merge of a split cache) must catch plausible
mistakes in them.  Each case plants one mistake in a copy of the oracle
package (on the CPU, in a temporary directory) and runs the matching pin file
against it; it must fail.  The unmodified oracle passes those files itself.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "oracle")

MUTANTS = [
    ("topk_ties_high_column_first", "order = np.lexsort((cols, -x))[:k]",
     "order = np.lexsort((-cols, -x))[:k]", "test_oracle_topk_pins.py"),
    ("topk_nan_not_minus_inf", "        x[np.isnan(x)] = -np.inf\n        order", "        order",
     "test_oracle_topk_pins.py"),
    ("sampling_ignores_temperature", "np.exp((x - x[0]) / temperature)", "np.exp(x - x[0])",
     "test_oracle_topk_pins.py"),
    ("rope_sign_flipped", "[x1 * c - x2 * s, x2 * c + x1 * s]", "[x1 * c + x2 * s, x2 * c - x1 * s]",
     "test_oracle_rope_pins.py"),
    ("rope_frequency_exponent", "(-2.0 * np.arange(half, dtype=np.float64) / d)",
     "(-1.0 * np.arange(half, dtype=np.float64) / d)", "test_oracle_rope_pins.py"),
    ("window_one_key_too_many", "lo = max(0, i - window + 1)", "lo = max(0, i - window)",
     "test_oracle_window_pins.py"),
    ("partial_wrong_log_base", "s = (k @ q) * float(scale) / np.log(2.0)",
     "s = (k @ q) * float(scale) * np.log(2.0)", "test_keysplit_cpu.py"),
    ("merge_natural_weights", "w = [0.0 if m == -np.inf else 2.0 ** (m - M) for m, _, _ in parts]",
     "w = [0.0 if m == -np.inf else np.exp(m - M) for m, _, _ in parts]", "test_keysplit_cpu.py"),
]


def _run_pins(tmp_path, pins, old=None, new=None):
    dst = tmp_path / "oracle"
    shutil.copytree(PKG, dst, ignore=shutil.ignore_patterns("__pycache__"))
    init = dst / "__init__.py"
    src = init.read_text()
    if old is not None:
        assert src.count(old) == 1, "mutation anchor not found once"
        src = src.replace(old, new)
    # a marker the pins' process can see: proves the copy is the one imported
    init.write_text(src + "\nPLANTED_COPY = True\n")
    env = dict(os.environ, RSWA_ORACLE_DIR=str(tmp_path), OMP_NUM_THREADS="1")
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           "-k", "not gloo", os.path.join(ROOT, "tests", pins)],
                          env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)


@pytest.fixture(scope="module")
def runs(tmp_path_factory):
    """The control run and every mutant's pin run, side by side."""
    import concurrent.futures as cf
    jobs = [("control", None, None, "test_oracle_rope_pins.py")] + list(MUTANTS)
    with cf.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
        futs = {name: ex.submit(_run_pins, tmp_path_factory.mktemp(name), pins, old, new)
                for name, old, new, pins in jobs}
        return {k: f.result() for k, f in futs.items()}


@pytest.mark.slow
def test_unplanted_copy_passes_and_is_the_one_imported(runs, tmp_path):
    r = runs["control"]
    assert r.returncode == 0, r.stdout[-2000:]
    dst = tmp_path / "oracle"
    shutil.copytree(PKG, dst, ignore=shutil.ignore_patterns("__pycache__"))
    init = dst / "__init__.py"
    init.write_text(init.read_text() + "\nPLANTED_COPY = True\n")
    env = dict(os.environ, RSWA_ORACLE_DIR=str(tmp_path))
    probe = subprocess.run([sys.executable, "-c",
                            "import sys, os; sys.path.insert(0, os.environ['RSWA_ORACLE_DIR']); "
                            "import oracle; print(getattr(oracle, 'PLANTED_COPY', False))"],
                           env=env, cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert probe.stdout.strip() == "True"


@pytest.mark.slow
@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_pins_catch_python_mutant(runs, name):
    r = runs[name]
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout, r.stdout[-2000:]  # a failing pin, not a broken import
