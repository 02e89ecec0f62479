import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


_CUDA = None


def pytest_runtest_setup(item):
    """GPU tests skip before doing any work when no CUDA device is present."""
    global _CUDA
    if "gpu" in item.keywords:
        if _CUDA is None:
            try:
                import torch
                _CUDA = torch.cuda.is_available()
            except Exception:
                _CUDA = False
        if not _CUDA:
            pytest.skip("no CUDA device")
