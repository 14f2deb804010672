import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(autouse=True)
def _bounds_checked_build():
    """Under the bounds-checked debug build (CF_LIBRARY=debug) every test
    must leave no failed index check behind."""
    yield
    if os.environ.get("CF_LIBRARY") == "debug":
        from activation_residual_compression_cf_b200 import cf
        hit = cf.cf_debug_bounds_take()
        assert hit == 0, f"index check failed: tag {hit >> 16:#x}, line {hit & 0xffff}"
