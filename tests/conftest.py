import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU-side oracle runs")


def load_golden(name):
    """Parse a golden text fixture: 'key v1 v2 ...' and 'key idx: v1 v2 ...' lines."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(None, 1) if " " in line else (line, "")
            if ":" in rest:
                idx, vals = rest.split(":", 1)
                out.setdefault(key, {})[int(idx)] = [int(x) for x in vals.split()]
            else:
                out[key] = [int(x) for x in rest.split()]
    return out
