import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200) and the built libfq.so")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def read_golden(name):
    """Rows of a whitespace-separated golden file, comments (#...) stripped."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


@pytest.fixture(autouse=True, scope="module")
def _no_bounded_wait_gave_up(request):
    """After every GPU test module: no kernel of the library gave up a bounded wait (a timed-out
    wait leaves unspecified outputs, so parity alone could miss it)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import random_access_kv_fq_b200 as fq
    n = fq.fq_wait_status(clear=True)
    assert n == 0, f"{n} CTAs gave up a bounded wait during {request.node.name}"
