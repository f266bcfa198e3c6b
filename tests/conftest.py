import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_sessionfinish(session, exitstatus):
    path = os.environ.get("SAGE_PARITY_REPORT")
    if not path:
        return
    try:
        from _helpers import REPORT
    except Exception:
        return
    if REPORT:
        import json
        with open(path, "w") as f:
            json.dump(REPORT, f, indent=0)
