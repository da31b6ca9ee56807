import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an NVIDIA B200 (sm_100a); runs the CUDA path")
    config.addinivalue_line("markers", "slow: full-size parity case (seconds to minutes)")


@pytest.fixture(scope="session")
def lib_path():
    """Path of the built librkv.so, building it in-tree if it is missing."""
    from rolling_kv_cache_rope_b200 import build as b
    return b.ensure_built()
