import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built libdsa.so")
    config.addinivalue_line("markers", "slow: full-size oracle runs (seconds to minutes of CPU)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()
