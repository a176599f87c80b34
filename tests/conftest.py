import os
import sys

import pytest

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if REPO not in sys.path:
    sys.path.insert(0, REPO)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes of CPU oracle work)")


@pytest.fixture(scope="session", autouse=True)
def _built_generators():
    """The seeded generators are compiled in-tree; build them once if missing."""
    import synth
    if not (os.path.exists(synth.HOST_LIB) and os.path.exists(synth.DEV_LIB)):
        synth.build()
    yield
