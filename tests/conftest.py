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
    """Parse a whitespace fixture: '# ...' comments, then 'key v1 v2 ...' lines.
    Returns {key: [list of rows of floats]}."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            conv = []
            for v in vals:
                try:
                    conv.append(float(v))
                except ValueError:
                    conv.append(v)
            out.setdefault(key, []).append(conv)
    return out


@pytest.fixture(scope="session")
def golden():
    return read_golden
