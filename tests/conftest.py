import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built libcce.so")
    config.addinivalue_line("markers", "slow: full-size cases (minutes of oracle time)")


@pytest.fixture(scope="session", autouse=True)
def _built_library():
    """Build libcce.so in-tree if it is missing or older than its sources."""
    from linear_cross_entropy_cce_b200 import build
    if build.needs_build():
        build.build()
    yield
