import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session", autouse=True)
def _build_libraries():
    """Build the CPU oracle and the CUDA library in-tree when missing or stale
    (nvcc cross-compiles for sm_100a without a GPU)."""
    import oracle
    from dynamic_expert_routing_router_b200 import build
    oracle.build()
    build.build()
