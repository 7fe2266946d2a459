import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    # the CUDA library, the device table filler and the C oracle, built in-tree if missing or
    # older than their sources (nvcc cross-compiles sm_100a without a GPU)
    import __graft_entry__
    __graft_entry__.build_libraries()
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity cases (minutes)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    return oracle
