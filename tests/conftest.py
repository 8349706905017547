import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running full-size case")
    # tests/test_oracle_mutations.py runs the oracle pins in a child process with one
    # planted oracle mistake named here
    mutation = os.environ.get("DSA_ORACLE_MUTATION")
    if mutation:
        from tests import oracle_mutations
        oracle_mutations.apply(mutation)


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
