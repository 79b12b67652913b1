import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: longer CPU test")
    config.addinivalue_line("markers", "late: long full-size parity run, ordered after the other tests")


def pytest_collection_modifyitems(config, items):
    # Long full-size parity runs go last (a stable sort keeps the rest in order),
    # so quicker failures surface first.
    items.sort(key=lambda it: it.get_closest_marker("late") is not None)
