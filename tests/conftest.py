import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU oracle case")
    config.addinivalue_line("markers", "sets_faults: deliberately sets device fault bits (and clears them)")


@pytest.fixture(autouse=True)
def _no_device_faults(request):
    """After every GPU test: no bounded device wait may have given up."""
    yield
    if request.node.get_closest_marker("gpu") is None or request.node.get_closest_marker("sets_faults"):
        return
    import torch
    if not torch.cuda.is_available():
        return
    import implicit_long_convolution_b200 as hy
    faults = hy.device_faults(clear=True)
    assert faults == 0, "device fault bits 0x%x after %s" % (faults, request.node.nodeid)


def pytest_sessionfinish(session, exitstatus):
    path = os.environ.get("PARITY_LOG")
    if not path:
        return
    try:
        import json
        import _helpers
        with open(path, "w") as f:
            json.dump(_helpers.RECORD, f, indent=1)
    except Exception:
        pass
