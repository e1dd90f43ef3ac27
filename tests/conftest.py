import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built libtq.so")
    config.addinivalue_line("markers", "slow: longer CPU test")


def load_golden(name):
    """Parse a tests/golden/*.txt fixture: key -> (list of str values, tolerance)."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            out[parts[0]] = (parts[1:-1], float(parts[-1]))
    return out
