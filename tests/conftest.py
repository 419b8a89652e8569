import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def golden():
    import json
    with open(os.path.join(ROOT, "tests", "golden", "page_numbers.json")) as f:
        return json.load(f)


@pytest.fixture(autouse=True)
def _device_status_checked(request):
    """GPU tests run with the binding reading back the device status word
    after every forward and backward call: a bounded wait that ran out
    inside a kernel (leaving a tile unwritten) turns the test red."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    import bit_nf4_quantized_09_b200 as q
    q.set_check_device_status(True)
    try:
        yield
    finally:
        q.set_check_device_status(True)
