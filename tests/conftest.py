import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size oracle runs (seconds to a minute each)")


def pytest_collection_modifyitems(config, items):
    # A GPU test that does not finish in time ends its own process (the watchdog
    # thread exits it, which also releases the CUDA context), instead of holding
    # the GPU until an outer limit.
    for item in items:
        if item.get_closest_marker("gpu") and not item.get_closest_marker("timeout"):
            item.add_marker(pytest.mark.timeout(600, method="thread"))
