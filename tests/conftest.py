import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (minutes)")


def read_sections(name):
    """Parse a golden fixture: '# comments', '[section]' headers, whitespace rows."""
    sections, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("[") and line.endswith("]"):
                cur = line[1:-1]
                sections[cur] = []
                continue
            if cur is None:
                sections.setdefault("", []).append(line.split())
            else:
                sections[cur].append(line.split())
    return sections


@pytest.fixture(scope="session")
def golden():
    return read_sections
