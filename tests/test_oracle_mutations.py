"""Each plausible mistake planted in the oracle (tests/oracle_mutations.py) makes at least
one oracle pin fail, and the unmutated copies of the replaced functions pass them all.
The pins run in a child process per case on the CPU, several cases at a time."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

from tests.oracle_mutations import CONTROLS, MUTATIONS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_pins(name):
    env = dict(os.environ, DSA_ORACLE_MUTATION=name, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1",
               MKL_NUM_THREADS="1")
    p = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q", "-m", "not gpu",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return p.returncode, p.stdout[-1500:] + p.stderr[-1500:]


@pytest.fixture(scope="module")
def outcomes():
    names = sorted(MUTATIONS) + sorted(CONTROLS)
    workers = max(1, min(8, os.cpu_count() or 1))
    with ThreadPoolExecutor(workers) as ex:
        return dict(zip(names, ex.map(_run_pins, names)))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(outcomes, name):
    rc, out = outcomes[name]
    assert rc == 1 and " failed" in out, out


@pytest.mark.parametrize("name", sorted(CONTROLS))
def test_pins_pass_unmutated_copies(outcomes, name):
    rc, out = outcomes[name]
    assert rc == 0, out
