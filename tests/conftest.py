import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_sessionfinish(session, exitstatus):
    """Write the recorded GPU comparison margins (one JSON line each) when
    MTLA_PARITY_LOG names a file."""
    path = os.environ.get("MTLA_PARITY_LOG")
    if not path:
        return
    import json
    import sys
    harness = sys.modules.get("gpu_harness")
    if harness is None:
        return
    with open(path, "w") as f:
        for test, rel, elem in harness.MARGINS:
            f.write(json.dumps({"test": test, "rel": rel, "elem": elem}) + "\n")
