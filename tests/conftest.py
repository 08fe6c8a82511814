import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU case")


def load_golden(name):
    """Parse a tests/golden fixture: name value tol | citation."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0] if line.lstrip().startswith("#") else line
            if not line.strip():
                continue
            head, _, cite = line.partition("|")
            key, val, tol = head.split()
            out[key] = (float(val), float(tol), cite.strip())
    return out
