import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built libkdn.so")


def cuda_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def kdn():
    """The CUDA binding; GPU tests fail loudly if the device or the library is missing."""
    import torch
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    from kalman_delta_rule_b200 import binding
    return binding


def pytest_sessionfinish(session, exitstatus):
    """Write every parity check's achieved error to $KDN_PARITY_LOG (JSON), if set."""
    path = os.environ.get("KDN_PARITY_LOG")
    if not path:
        return
    import json
    from tests.kdn_testutil import MARGINS
    os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
    with open(path, "w") as f:
        json.dump(MARGINS, f, indent=0)
