import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name: str) -> dict:
    """Parse a ``key = value`` fixture under tests/golden (``#`` starts a comment)."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = (p.strip() for p in line.split("=", 1))
            out[k] = v
    return out


def num(v: str) -> float:
    """A fixture number, allowing a plain quotient such as ``50/127``."""
    if "/" in v:
        a, b = v.split("/")
        return float(a) / float(b)
    return float(v)


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle
