import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Parse a golden fixture: '#' comments, 'key = value' lines, blank-line separated records."""
    records, cur = [], {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                if cur:
                    records.append(cur)
                    cur = {}
                continue
            key, _, val = line.partition("=")
            cur[key.strip()] = val.strip()
    if cur:
        records.append(cur)
    return records


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle
