import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def da_lib():
    """The CUDA library, built in-tree if missing (nvcc cross-compiles without a GPU)."""
    from variable_length_paged_b200 import build, da
    build.build()
    da.lib()
    return da


def cuda_available() -> bool:
    import torch
    return torch.cuda.is_available()
