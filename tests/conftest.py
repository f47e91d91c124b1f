import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_library():
    """Build libsdq.so (and the oracle) before any test imports the package;
    a no-op when they are up to date."""
    import __graft_entry__
    __graft_entry__._build_module().build()
    import oracle
    oracle.build()


def pytest_configure(config):
    _build_library()
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a); runs the CUDA path")
    config.addinivalue_line("markers", "slow: full-size case (minutes of CPU time)")


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
