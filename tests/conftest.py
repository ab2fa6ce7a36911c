import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200) and the built library")


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


@pytest.fixture(autouse=True)
def _debug_build_reports_no_bounds_failure(request):
    """With LH_LIBRARY=debug (the bounds-checking build), every GPU test must end
    without a bounds failure in the device status; the status is cleared first."""
    if os.environ.get("LH_LIBRARY") != "debug" or "gpu" not in request.keywords:
        yield
        return
    from long_context_lh_b200 import lighthouse as lh
    lh.lh_read_device_status()
    yield
    code = lh.lh_read_device_status()
    assert code & lh.LH_STATUS_BOUNDS == 0, f"bounds check failed: status {code:#x}"


def pytest_report_header(config):
    if os.environ.get("LH_LIBRARY") == "debug":
        from long_context_lh_b200 import lighthouse as lh
        return f"library under test: {os.path.basename(lh.LIB_PATH)}"
    return None
