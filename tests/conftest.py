import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")


def pytest_sessionfinish(session, exitstatus):
    """Write every parity error measured in this session to $GRET_PARITY_LOG (JSON), if set."""
    path = os.environ.get("GRET_PARITY_LOG")
    if not path:
        return
    import json
    try:
        from parity import ERRORS
    except ImportError:
        return
    with open(path, "w") as f:
        json.dump(ERRORS, f, indent=0)


@pytest.fixture(scope="session")
def oracle_mod():
    from oracle import oracle
    oracle.lib()
    return oracle
