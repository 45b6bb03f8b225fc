import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def load_golden(name):
    """Parse a golden fixture: 'key: numbers' lines, ';' separates matrix rows."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(":")
            rows = [[float(v) for v in r.split()] for r in val.split(";")]
            out[key.strip()] = rows[0] if len(rows) == 1 else rows
    return out


@pytest.fixture
def golden():
    return load_golden
