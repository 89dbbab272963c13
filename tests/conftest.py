import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


def load_golden(name):
    """Parse a tests/golden/*.txt file -> (n, input uint16 list, container bytes)."""
    path = os.path.join(ROOT, "tests", "golden", name)
    n = None
    inp = []
    cont = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1)
            if key == "n":
                n = int(val)
            elif key == "input":
                inp += [int(t, 16) for t in val.split()]
            elif key == "container":
                cont += [int(t, 16) for t in val.split()]
    return n, inp, bytes(cont)


@pytest.fixture(scope="session")
def golden_names():
    d = os.path.join(ROOT, "tests", "golden")
    return sorted(f for f in os.listdir(d) if f.endswith(".txt"))
