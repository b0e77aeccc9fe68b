"""Shared test configuration: the ``gpu`` marker and import paths.

Tests marked ``gpu`` need a CUDA device (a B200) and call the library through its C ABI;
everything else runs on the CPU (oracle pins, host-side validation, symbol exports, gloo ranks).
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libtp.so")


def pytest_collection_modifyitems(config, items):
    # GPU tests need a CUDA device; on a host without one they are skipped (CPU runs select
    # -m "not gpu" anyway), so that a plain `pytest tests` still works there.
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device visible")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
