import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def read_golden(name):
    """Parse a tests/golden fixture: 'key: values' lines and 'key:' matrix blocks."""
    out, cur = {}, None
    with open(os.path.join(HERE, "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if ":" in line:
                key, rest = line.split(":", 1)
                vals = [float(v) for v in rest.split()]
                if vals:
                    out[key.strip()] = vals
                    cur = None
                else:
                    cur = key.strip()
                    out[cur] = []
            elif cur is not None:
                out[cur].append([float(v) for v in line.split()])
    return out
