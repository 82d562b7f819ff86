import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running statistical or full-size case")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def cuda_lib():
    """The C-ABI library through its Python binding; fails (never skips) without a GPU."""
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tree_verify_b200 import binding
    binding.load()
    return binding
