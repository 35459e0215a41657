import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running")


import pytest  # noqa: E402


@pytest.fixture(scope="session")
def dmuon_lib():
    """The built CUDA library (built in-tree on demand; nvcc cross-compiles)."""
    from newton_schulz_normalise_b200 import build
    build.build()
    from newton_schulz_normalise_b200 import binding
    return binding


def cuda_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False
