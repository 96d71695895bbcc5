"""Test configuration: the `gpu` marker and the shared fixtures.

Tests marked `gpu` need a CUDA device and the built GPU library; everything
else runs on the CPU (the oracle pins, host-side logic, the C-ABI symbol
check and the multi-process gloo tests).
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built libcskv.so")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def cskv_built():
    """Build libcskv.so in-tree if it is missing or stale (nvcc cross-compiles without a GPU)."""
    from compressed_sparse_kv_02_b200 import build
    return build.build()
