import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a) and the built "
                   "CUDA library")


def pytest_collection_modifyitems(config, items):
    # GPU tests fail loudly (not skip) when no device is present, so a GPU run
    # that silently lost its device cannot pass; the CPU suite deselects them
    # with -m "not gpu".
    pass
