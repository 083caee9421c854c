import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(scope="session", autouse=True)
def _built_libraries():
    """Compile the oracle (gcc) and the CUDA library (nvcc, sm_100a) in-tree
    when they are missing or older than their sources."""
    import oracle
    oracle.build()
    from scaled_dot_product_11_b200 import build as lib_build
    if lib_build.needs_build() and lib_build.nvcc_available():
        lib_build.build()
    yield
