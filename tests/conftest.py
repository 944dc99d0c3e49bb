import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload check")


@pytest.fixture(scope="session")
def golden():
    """Key/value facts printed by the method pages (tests/golden/page_facts.txt)."""
    facts = {}
    with open(os.path.join(ROOT, "tests", "golden", "page_facts.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            facts[key.strip()] = val.split()
    return facts
