import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size checks that take longer")


@pytest.fixture(scope="session")
def lib_path():
    """Path of the built C-ABI library; builds it (nvcc, sm_100a) if absent."""
    from exact_io_aware_78_b200 import build as _build
    return _build.ensure_built()
