import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libtern.so")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _no_failed_device_checks(request):
    """Under TERN_CHECK_DEVICE_STATUS=1 (set by test_debug_gpu for its runs against the TERN_DEBUG
    build), every GPU test must leave the sticky device status clean: no bounded wait ran out and no
    bounds check of the debug build failed."""
    yield
    if os.environ.get("TERN_CHECK_DEVICE_STATUS") != "1" or "gpu" not in request.keywords:
        return
    from ternary_weight_only_tern_b200 import _lib, api
    st = _lib.load().tern_device_status(api._stream())
    assert st == 0, f"device status after the test: {_lib.STATUS_NAMES.get(st, st)}"
