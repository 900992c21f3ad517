"""Shared pytest configuration: the ``gpu`` marker and the repository root on sys.path."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def lib():
    """The CUDA library through its Python binding (GPU tests only)."""
    if not cuda_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    from w4a8_codebook_quantized_rotate_b200 import binding
    return binding
