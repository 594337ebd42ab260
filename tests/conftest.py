import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU oracle run")


@pytest.fixture(scope="session", autouse=True)
def _built_host_libs():
    """The oracle and the input generator are host libraries; build them once per session."""
    import moe_inputs
    import oracle
    oracle.build()
    moe_inputs.build()
    yield
