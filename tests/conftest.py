import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def read_golden(name):
    """Parse a `key = v1 v2 ...` fixture; values are floats (ints where they parse)."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = (t.strip() for t in line.split("=", 1))
            vals = []
            for tok in v.split():
                try:
                    vals.append(int(tok))
                except ValueError:
                    vals.append(float(tok))
            out[k] = vals
    return out


@pytest.fixture
def golden():
    return read_golden
