import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


def read_golden(name):
    """Parses a tests/golden text fixture: '#' lines are comments, 'key value'
    lines are scalars and the remaining lines are integer rows."""
    meta, rows = {}, []
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0].isalpha():
                meta[parts[0]] = int(parts[1])
            else:
                rows.append([int(p) for p in parts])
    return meta, rows
