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
    # A GPU test on a machine without a GPU is a configuration error on the GPU machine, but on the
    # CPU box the driver selects -m "not gpu"; skip (do not fail) when no device is visible.
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device visible")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
