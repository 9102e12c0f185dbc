import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
for _p in (ROOT, os.path.join(ROOT, "tests")):
    if _p not in sys.path:
        sys.path.insert(0, _p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (runs the CUDA path through the C-ABI)")
    config.addinivalue_line("markers", "slow: long-running oracle comparison at full layer sizes")


@pytest.fixture(scope="session")
def lib():
    """The C-ABI library, loaded through the Python binding."""
    from host_offloaded_layer_b200 import _lib
    return _lib.load()
