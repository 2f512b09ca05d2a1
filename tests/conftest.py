import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Non-comment lines of a fixture under tests/golden/."""
    path = os.path.join(ROOT, "tests", "golden", name)
    with open(path, encoding="utf-8") as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def golden_table(name):
    out = {}
    for ln in read_golden(name):
        key, rest = ln.split("=", 1)
        out[key.strip()] = float(rest.split(";", 1)[0])
    return out
