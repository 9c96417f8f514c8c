import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) GPU")


def _read_fixture(name):
    path = os.path.join(ROOT, "tests", "golden", name)
    rows, kv = [], {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if "=" in line:
                k, v = line.split("=", 1)
                kv[k.strip()] = v.split()
            else:
                rows.append([int(t) for t in line.split()])
    return rows, kv


@pytest.fixture
def golden():
    return _read_fixture
