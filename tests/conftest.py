import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large CPU work (oracle at full size)")


def pytest_collection_modifyitems(config, items):
    import torch

    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


# KDA_PARITY_REPORT=<file>: write every parity check's error figure and its
# tolerance, per test, as JSON (the largest margin used is the number to watch).
_REPORT = {}


@pytest.fixture(autouse=True)
def _parity_record(request):
    yield
    if not os.environ.get("KDA_PARITY_REPORT") or "parity" not in sys.modules:
        return
    rec = sys.modules["parity"].RECORD
    if rec:
        _REPORT[request.node.nodeid] = [
            {"what": w, "mode": m, "error": e, "tol": t} for (w, m, e, t) in rec]
        rec.clear()


def pytest_sessionfinish(session, exitstatus):
    path = os.environ.get("KDA_PARITY_REPORT")
    if path and _REPORT:
        import json

        with open(path, "w") as f:
            json.dump(_REPORT, f, indent=1)
