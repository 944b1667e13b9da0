import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def read_golden(name):
    """Parse a tests/golden fixture: '#' comments, 'key: values' lines (repeated keys accumulate)."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if ":" in line:
                k, v = line.split(":", 1)
                out.setdefault(k.strip(), []).append(v.split())
            else:
                out.setdefault("_rows", []).append(line.split())
    return out


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle
