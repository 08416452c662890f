import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

_REPORT = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: exhaustive sweeps")


@pytest.fixture
def parity_report(request):
    """Record a parity test's worst error ratios; written as JSON to the path
    in IQK_PARITY_REPORT (if set) when the session ends."""
    def add(what, stats):
        _REPORT.append({"test": request.node.nodeid, "what": what, **stats})
    return add


def pytest_sessionfinish(session, exitstatus):
    path = os.environ.get("IQK_PARITY_REPORT")
    if path and _REPORT:
        with open(path, "w") as f:
            json.dump(_REPORT, f, indent=1)
