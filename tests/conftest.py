"""Shared pytest configuration.

Markers: ``gpu`` (needs a B200 and the built CUDA library) and ``slow``.
The CPU suite is ``pytest -m "not gpu"``; GPU parity is ``pytest -m gpu``.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running test")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


@pytest.fixture(autouse=True)
def _gpu_guard(request):
    """GPU tests need CUDA; without it they are skipped (they are deselected by
    ``-m "not gpu"`` anyway).  With CUDA present, a missing library fails."""
    if request.node.get_closest_marker("gpu") is not None:
        import torch
        if not torch.cuda.is_available():
            pytest.skip("no CUDA device")
