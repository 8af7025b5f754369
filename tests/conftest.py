import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def dvlm_lib():
    """The in-tree CUDA library, (re)built when a source changed."""
    from block_diffusion_vlm_b200 import build, lib
    build.build()
    return lib()


@pytest.fixture(scope="session")
def cuda(dvlm_lib):
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")
