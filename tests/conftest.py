import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a B200)")
    config.addinivalue_line("markers", "slow: full-size workload (minutes)")


@pytest.fixture(scope="session", autouse=True)
def _built_host_libs():
    """Build the host-side libraries (generator, oracle) if they are missing."""
    import oracle
    import synth

    if not os.path.exists(synth.HOST_LIB):
        synth.build()
    if not os.path.exists(oracle.LIB):
        oracle.build()
    yield
