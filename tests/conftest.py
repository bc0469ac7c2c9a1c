import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle

    oracle.load()
    return oracle


@pytest.fixture(scope="session")
def mxlib():
    """libmxscale built in-tree (nvcc cross-compiles without a GPU)."""
    from scale_factor_layout_b200 import _build, _binding

    _build.build()
    return _binding.lib()


def gpu_available():
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False
