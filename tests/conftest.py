import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: longer CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def dev():
    """The CUDA device for gpu-marked tests. There is no fallback: without a GPU
    these tests fail instead of silently testing something else."""
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("gpu-marked test run without a CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(scope="session")
def lib(dev):
    from precision_moe_numerics_quantize_b200 import nvfp4moe
    return nvfp4moe
