"""The oracle's pins catch plausible mistakes: each mistake of
tests/oracle_mutants.py, planted in the CPU oracle of a child process, must make
several pins of tests/test_oracle_pins.py fail, and with none planted they all
pass.  The children run side by side, one BLAS thread each."""
import concurrent.futures as cf
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.join(ROOT, "tests")
sys.path.insert(0, TESTS)
import oracle_mutants  # noqa: E402

# the pins a mutant must break at least this many of
MIN_FAILED = 2


def _run(name):
    env = dict(os.environ, MTA_ORACLE_MUTANT=name, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1",
               MKL_NUM_THREADS="1",
               PYTHONPATH=os.pathsep.join(p for p in (TESTS, ROOT, os.environ.get("PYTHONPATH")) if p))
    r = subprocess.run([sys.executable, "-m", "pytest", "-p", "oracle_mutants", "-p", "no:cacheprovider",
                        "-q", "-m", "not gpu", os.path.join(TESTS, "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    m = re.search(r"(\d+) failed", r.stdout)
    p = re.search(r"(\d+) passed", r.stdout)
    return r.returncode, int(m.group(1)) if m else 0, int(p.group(1)) if p else 0, r.stdout[-2000:]


@pytest.fixture(scope="module")
def results():
    names = ["none"] + sorted(oracle_mutants.MUTANTS)
    with cf.ThreadPoolExecutor(max_workers=min(len(names), max(2, os.cpu_count() or 2))) as ex:
        return dict(zip(names, ex.map(_run, names)))


def test_pins_pass_with_nothing_planted(results):
    rc, failed, passed, out = results["none"]
    assert rc == 0 and failed == 0 and passed > 0, out


@pytest.mark.parametrize("name", sorted(oracle_mutants.MUTANTS))
def test_planted_mistake_fails_several_pins(results, name):
    rc, failed, passed, out = results[name]
    assert rc == 1 and failed >= MIN_FAILED, (name, failed, out)
