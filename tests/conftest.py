import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")
    config.addinivalue_line("markers", "slow: full-size parity cases")


def pytest_collection_modifyitems(config, items):
    # A GPU test without a GPU is an error, never a silent skip into a
    # fallback: there is none.  Deselection is done with -m "not gpu".
    pass


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle
