import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a) and libwan.so")


def pytest_collection_modifyitems(config, items):
    # GPU tests cannot run on a machine without a CUDA device; skip them
    # there instead of failing (the CPU suite runs with -m "not gpu").
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def golden(key):
    """Values of one line of tests/golden/pages_numbers.txt."""
    path = os.path.join(ROOT, "tests", "golden", "pages_numbers.txt")
    with open(path, encoding="utf-8") as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, rest = line.split(":", 1)
            if k.strip() == key:
                vals = rest.split("|", 1)[0].split()
                return [float(v) for v in vals]
    raise KeyError(key)


@pytest.fixture
def gold():
    return golden
