import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")


def pytest_collection_modifyitems(config, items):
    # a GPU test that runs on a host without a GPU fails loudly instead of
    # silently falling back; selecting `-m "not gpu"` skips them.
    pass


@pytest.fixture(scope="session")
def oracle():
    import oracle as _o
    _o.build()
    return _o
