import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle

TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_sessionfinish(session, exitstatus):
    path = os.environ.get("PARITY_REPORT")
    if not path:
        return
    try:
        import json
        import parity
        with open(path, "w") as f:
            json.dump(parity.REPORT, f, indent=1)
    except Exception:  # noqa: BLE001 - reporting must not change the test outcome
        pass
