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
