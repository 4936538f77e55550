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


def load_build_module():
    """The package's build step, loaded by path (importing the package itself
    needs the built library)."""
    import importlib.util

    path = os.path.join(ROOT, "block_sparse_attention_frame_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_lvsa_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="session")
def lib():
    """The C-ABI library, built in-tree if it is missing or stale."""
    load_build_module().build_library(quiet=True)
    import block_sparse_attention_frame_b200 as lvsa

    return lvsa


@pytest.fixture(scope="session")
def gpu_lib(lib):
    if not cuda_available():
        pytest.fail("GPU test collected on a machine without CUDA")
    # a stuck pipeline gives up after 0.5 s per wait instead of 4 s
    lib.lvsa_set_wait_budget_ns(500_000_000)
    return lib
