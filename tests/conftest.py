import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libeqw.so")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def read_golden(name):
    """Non-comment lines of a golden fixture file."""
    with open(os.path.join(GOLDEN, name)) as fh:
        return [ln.strip() for ln in fh if ln.strip() and not ln.lstrip().startswith("#")]


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle
