import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running full-size case")


def pytest_sessionstart(session):
    # The shared library is git-ignored; build it (in-tree, sm_100a) when missing or stale.
    from recurrent_state_serving_b200 import build
    build.build()
