import json
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


def pytest_sessionfinish(session, exitstatus):
    """With BEAM_PARITY_REPORT=<path>, write what the parity tests observed
    (router logit error, decision flip rate, worst value errors) as JSON."""
    path = os.environ.get("BEAM_PARITY_REPORT")
    mod = sys.modules.get("_parity")
    if not path or mod is None:
        return
    with open(path, "w") as f:
        json.dump(mod.REPORT, f, indent=1)
