import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")
    config.addinivalue_line("markers", "status_checked: GPU test that reads the device status itself")


@pytest.fixture(autouse=True)
def _device_status_clean(request):
    """Every GPU test must leave the library's device status clean (no wait timed out, no
    index out of range) unless it checks the status itself."""
    yield
    if request.node.get_closest_marker("gpu") is None or request.node.get_closest_marker("status_checked"):
        return
    from bit_block_scaled_nvfp4_b200 import api
    st = api.check_status()
    assert st == 0, f"device status {st} after {request.node.name}"
