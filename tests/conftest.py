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
    """Parse a golden fixture: '# ...' comment lines, 'key: value' lines and
    bare whitespace-separated rows.  Returns (dict, rows)."""
    kv, rows = {}, []
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
            else:
                rows.append(line.split())
    return kv, rows


@pytest.fixture(scope="session")
def golden():
    return read_golden
