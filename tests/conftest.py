import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def cuda_available() -> bool:
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def lib():
    """The C-ABI library, built in-tree if it is missing or stale."""
    from block_sparse_attention_frame_b200 import build as libbuild

    libbuild.build_library(quiet=True)
    import block_sparse_attention_frame_b200 as lvsa

    return lvsa


@pytest.fixture(scope="session")
def gpu_lib(lib):
    if not cuda_available():
        pytest.fail("GPU test collected on a machine without CUDA")
    return lib
