import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Parse a tests/golden fixture: 'key = value' lines and bare CSV rows."""
    path = os.path.join(ROOT, "tests", "golden", name)
    kv, rows = {}, []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if "=" in line:
                k, v = (s.strip() for s in line.split("=", 1))
                kv[k] = v
            else:
                rows.append([s.strip() for s in line.split(",")])
    return kv, rows


@pytest.fixture
def golden():
    return read_golden
