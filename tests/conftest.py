import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    # GPU tests are selected with -m gpu / -m "not gpu". Without a device
    # they fail instead of skipping, so a machine whose GPU cannot be used
    # never reports a green GPU run.
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def golden_rows(name):
    """Rows of a whitespace-separated fixture under tests/golden/, comments dropped."""
    path = os.path.join(ROOT, "tests", "golden", name)
    rows = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle
