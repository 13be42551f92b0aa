import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built libfp4mx.so")
    config.addinivalue_line("markers", "slow: full-size workload (runs on the GPU box)")


def golden_rows(name):
    """Non-comment, non-empty lines of a golden fixture, split on whitespace."""
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


@pytest.fixture(scope="session")
def cuda():
    """The CUDA device for GPU tests: a missing GPU is a failure, never a silent skip."""
    import torch
    assert torch.cuda.is_available(), "GPU test run without a visible CUDA device"
    import block_scaled_fp4_amax_b200 as fp4
    fp4.lib()
    return torch.device("cuda:0")
