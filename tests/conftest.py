import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Parse a tests/golden/*.txt file of 'key value [tol]' lines into {key: (value, tol)}."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            out[parts[0]] = (float(parts[1]), float(parts[2]) if len(parts) > 2 else 0.0)
    return out


@pytest.fixture(scope="session")
def golden_rule():
    return read_golden("tara_rule_pages.txt")
