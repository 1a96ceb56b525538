import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")
    config.addinivalue_line("markers", "slow: full-size workload parity (minutes)")


@pytest.fixture(scope="session", autouse=True)
def _library_built():
    """Build librola.so once if it is missing (nvcc cross-compiles; no GPU needed)."""
    from sparse_rank_attention_b200 import LIB_PATH
    if not os.path.exists(LIB_PATH):
        from sparse_rank_attention_b200 import build
        build.build()
