import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # GPU tests on a machine without a GPU fail loudly at the first CUDA call;
    # they are deselected with -m "not gpu" there.
    pass


@pytest.fixture(scope="session")
def ora():
    import oracle
    oracle.build()
    return oracle
