import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")
    config.addinivalue_line("markers", "slow: long-running case")


def pytest_collection_modifyitems(config, items):
    """GPU-marked tests fail loudly (not skip) when selected without a GPU, so a GPU run
    can never pass silently on a machine that cannot execute the kernels."""
    return


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN
