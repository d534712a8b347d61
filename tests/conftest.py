"""Shared pytest set-up: the ``gpu`` marker, import paths and build fixtures."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a); run with -m gpu")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.load()


@pytest.fixture(scope="session")
def native_lib_path():
    """Path of the built C-ABI shared library (built on demand: nvcc cross-compiles
    without a GPU)."""
    from ffn_gated_activation_b200 import _build
    return _build.build_library()


@pytest.fixture(scope="session")
def cuda_device():
    """Fails (never skips) when CUDA is missing: a gpu-marked test must not pass
    without running the native path."""
    import torch
    assert torch.cuda.is_available(), "gpu-marked test needs a CUDA device"
    return torch.device("cuda", 0)
