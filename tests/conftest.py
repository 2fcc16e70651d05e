import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session", autouse=True)
def _built_oracle():
    from oracle.build_oracle import build_oracle
    build_oracle()
    yield


def load_golden(name):
    """Parse a tests/golden/*.txt fixture: '# ...' comments, 'key: values'."""
    path = os.path.join(ROOT, "tests", "golden", name)
    out = {}
    with open(path, encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.split()
    return out
