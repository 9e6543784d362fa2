import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU oracle work")


@pytest.fixture(scope="session", autouse=True)
def _built_libraries():
    """Compile libkda.so (nvcc, sm_100a) and the oracle (gcc) when stale."""
    from gated_delta_rule_139_b200 import build as kda_build
    import oracle
    kda_build.build()
    oracle.build()
