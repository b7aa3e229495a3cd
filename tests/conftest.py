"""Shared pytest configuration.

Tests marked ``gpu`` need a CUDA device (a B200) and the built library; they
are the parity tests proper and call the CUDA path through its C ABI.  All
other tests run on CPU: the oracle against its pins, the host allocator, host
argument validation, the exported-symbol check and the multi-process plumbing.
"""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
