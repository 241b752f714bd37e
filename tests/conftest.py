import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU (runs the CUDA path)")


def read_golden(name):
    """Parse a tests/golden fixture: '# ...' comments, 'case ...' headers, data lines."""
    path = os.path.join(ROOT, "tests", "golden", name)
    cases, cur = [], None
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case"):
                cur = {"head": line.split()[1:], "rows": []}
                cases.append(cur)
            else:
                cur["rows"].append(line)
    return cases


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle
