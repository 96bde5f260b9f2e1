import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_sessionfinish(session, exitstatus):
    """Writes the parity errors measured by the GPU tests to the file named
    by FLARE_PARITY_LOG (nothing when it is unset)."""
    path = os.environ.get("FLARE_PARITY_LOG")
    if not path:
        return
    try:
        import gpu_util
    except ImportError:
        return
    import json
    with open(path, "w") as f:
        json.dump(gpu_util.RECORDS, f, indent=0)
