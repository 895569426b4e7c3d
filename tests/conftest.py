import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size cases (minutes)")


def read_golden(name):
    """Parse a golden fixture: '# ...' comments, 'key: value' headers, and
    whitespace-separated data rows."""
    header, rows = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if ":" in line:
                k, v = line.split(":", 1)
                header[k.strip()] = v.strip()
            else:
                rows.append(line.split())
    return header, rows


@pytest.fixture
def golden():
    return read_golden
