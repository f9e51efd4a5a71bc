import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")


def golden(name: str):
    """Rows of a golden fixture as {key: (value_text, citation)}."""
    path = os.path.join(ROOT, "tests", "golden", name)
    rows = {}
    with open(path) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            key, value, cite = line.rstrip("\n").split("\t")
            rows[key] = (value, cite)
    return rows


@pytest.fixture(scope="session")
def page_numbers():
    return golden("page_numbers.txt")
