import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")


@pytest.fixture(autouse=True)
def _device_error_checks(request):
    """GPU tests run with the library's debug checks on: every call synchronises and
    turns a recorded bad index or timed-out wait into an exception; afterwards the
    device error word must be clear."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    import paged_kv_cache_442_b200 as pa
    from paged_kv_cache_442_b200 import build as pa_build
    pa_build.build()
    pa.pa_set_debug_checks(True)
    try:
        yield
    finally:
        pa.pa_set_debug_checks(False)
    assert pa.pa_check_device_errors() == 0
