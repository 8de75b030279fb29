import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a); parity against the CPU oracle")


@pytest.fixture(autouse=True)
def _no_expired_waits(request):
    """Every GPU test ends with no bounded device wait having given up (a wait
    that gives up leaves that launch's outputs undefined)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import hadamard_incoherence_transforms_b200 as hit

    assert hit.wait_timeouts(reset=True) == 0, "a bounded device wait gave up during this test"
