import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")


def pytest_collection_modifyitems(config, items):
    # Keep the file that must run last at the end, whatever the collection order.
    last = [it for it in items if os.path.basename(str(it.fspath)).startswith("test_zz_")]
    rest = [it for it in items if not os.path.basename(str(it.fspath)).startswith("test_zz_")]
    items[:] = rest + last
