import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


@pytest.fixture(scope="session")
def lib_path():
    """Path of the in-tree C-ABI library, building it first if it is missing."""
    from scaled_dot_product_12_b200 import build as _build
    path = _build.library_path()
    if not os.path.exists(path) or _build.is_stale():
        _build.build()
    return path
