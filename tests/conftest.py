"""Shared pytest setup: repository root on sys.path and the ``gpu`` marker.

Tests marked ``gpu`` need a CUDA device and the built CUDA library; they fail
(never skip) when either is missing, so a GPU run cannot pass vacuously.
"""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU and the built CUDA library")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for gpu-marked tests")
    return torch.device("cuda:0")
