import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def lib():
    """The native library, built in-tree if it is missing, loaded through the binding."""
    from w4a4_post_quantization_serq_b200 import _native, build
    if not os.path.exists(_native.LIB_PATH):
        build.build()
    return _native.load()
