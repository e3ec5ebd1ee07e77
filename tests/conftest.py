import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.fixture(scope="session")
def cuda_dev():
    """The CUDA device for -m gpu tests.  Fails (does not skip) without one:
    a GPU test that silently skips would hide a missing native path."""
    import torch
    assert torch.cuda.is_available(), "gpu test selected but no CUDA device is visible"
    return torch.device("cuda:0")


@pytest.fixture(scope="session")
def crs():
    """The product binding; importing it loads libcrs.so or raises."""
    import content_routed_sparse_b200 as m
    return m
