"""The oracle's pins catch plausible mistakes.

For every mistake planted in the oracle (tests/oracle_mutants.py: a
transposed S, the wrong importance region, a dropped count weight, the
wrong tie rule, sharp and flat swapped, the pooled query instead of the
token, a wrong pooling divisor or scale, a missing softmax term in the
backward, a RoPE sign ...), the oracle's pin tests are run against the
changed oracle in a child process and at least one of them must fail.  The
control loads the unchanged source through the same path and must pass.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

from oracle_mutants import MUTANTS

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)
PIN_FILES = ["tests/test_oracle.py", "tests/test_oracle_backward.py", "tests/test_oracle_coarse.py"]


def run_pins(name: str):
    env = dict(os.environ, ORACLE_MUTANT=name, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1",
               MKL_NUM_THREADS="1")
    env["PYTHONPATH"] = os.pathsep.join(p for p in (TESTS, ROOT, os.environ.get("PYTHONPATH", "")) if p)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "oracle_mutants", "-p", "no:cacheprovider",
           "-m", "not gpu", *PIN_FILES]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, (r.stdout + r.stderr)[-4000:]


@pytest.fixture(scope="module")
def outcomes():
    names = ["none", *sorted(MUTANTS)]
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        return dict(zip(names, ex.map(run_pins, names)))


def test_control_passes(outcomes):
    rc, out = outcomes["none"]
    assert rc == 0, out


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(outcomes, name):
    rc, out = outcomes[name]
    # exit code 1: tests ran and one failed (2-5 would be a broken run)
    assert rc == 1 and " failed" in out, (name, rc, out)
