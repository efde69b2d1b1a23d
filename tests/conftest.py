import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built libbatq")


@pytest.fixture(scope="session")
def lib():
    """The loaded C-ABI library (GPU tests only)."""
    from mxfp4_w4a4_post_block_b200 import _lib
    return _lib.load()


def pytest_sessionfinish(session, exitstatus):
    """With BATQ_PARITY_REPORT set to a path, write the code/scale mismatch counts of every
    quantiser parity check of the session there (JSON, by check label)."""
    path = os.environ.get("BATQ_PARITY_REPORT")
    if not path:
        return
    try:
        import parity
    except ImportError:
        return
    import json
    with open(path, "w") as f:
        json.dump(parity.REPORT, f, indent=1, sort_keys=True)
