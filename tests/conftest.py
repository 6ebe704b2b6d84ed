import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running oracle case")


def read_golden(name):
    """Parse a tests/golden/*.txt fixture: 'key: values' lines, '#' comments, '/' row breaks."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.strip()
    return out


def parse_matrix(v, conv=float):
    return [[conv(t) for t in row.split()] for row in v.split("/")]


def parse_vector(v, conv=float):
    return [conv(t) for t in v.split()]
