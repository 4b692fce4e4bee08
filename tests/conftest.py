import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Parse a tests/golden/*.txt fixture: '#' lines are comments, other lines are
    'key v1 v2 ...'.  Repeated keys are returned as a list of rows in file order."""
    import numpy as np

    rows = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.setdefault(key, []).append(np.array([float(v) for v in vals]))
    return rows


@pytest.fixture
def golden():
    return read_golden
