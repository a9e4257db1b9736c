import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running full-size case")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="session")
def ctx():
    """A library context on cuda:0 (GPU tests only)."""
    import torch
    from post_quantization_expert_b200 import clha
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    c = clha.Context(0)
    yield c
    torch.cuda.synchronize()
    c.close()
