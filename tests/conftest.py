import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def _ensure_library():
    """Build libkda_prefill.so in-tree when it is missing or stale (nvcc is on both machines)."""
    try:
        from kda_chunked_recurrent_b200 import build as _b
        if _b.needs_build():
            _b.build()
    except Exception as e:  # pragma: no cover - surfaced by the tests that need the library
        print(f"[conftest] library build failed: {e}")


_ensure_library()
