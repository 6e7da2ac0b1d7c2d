import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def ensure_library():
    """Build libmoe_b200.so in-tree if it is missing (a fresh checkout: the library is not
    committed).  nvcc cross-compiles for sm_100a without a GPU."""
    lib = os.path.join(ROOT, "mixture_experts_layer_50_b200", "libmoe_b200.so")
    if not os.path.exists(lib):
        from mixture_experts_layer_50_b200 import build
        build.build()
    return lib


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built library")
    # the test modules import the binding, which refuses to load without the library
    ensure_library()


@pytest.fixture(scope="session")
def cuda_dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
