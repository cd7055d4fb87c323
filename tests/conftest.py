import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture
def testing_lib():
    """Run the test against the test build of the library (the same kernels
    plus the forcing knobs and the fault injection); knobs are reset and the
    build's plan cache released afterwards."""
    from elementwise_optimizer_b200 import binding as B
    with B.testing_library() as L:
        yield L
