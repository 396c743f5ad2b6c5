import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")


def parse_golden(name):
    """Records of a golden text fixture: list of (kind, {key: value-string})."""
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kind, *fields = line.split()
            rec = {}
            for fld in fields:
                k, v = fld.split("=", 1)
                rec[k] = v
            out.append((kind, rec))
    return out


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()
