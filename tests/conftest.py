"""Shared pytest configuration.

Markers: ``gpu`` — needs a CUDA device (a B200); everything else runs on the CPU.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: test needs a CUDA GPU (sm_100a)")


@pytest.fixture(scope="session", autouse=True)
def _built_library():
    """Build libla_b200.so (in-tree, sm_100a) once per session if a source is newer, and make the
    tensor conveniences check the device status word after every call, so that a device-side
    error (a scan timeout) fails the test instead of leaving unwritten outputs."""
    from long_context_attention_la_b200 import build, la
    build.build()
    la.CHECK_STATUS = True


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
