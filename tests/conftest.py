import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large CPU work (still run by default)")


def pytest_sessionstart(session):
    """Build libspattn.so in-tree if it is missing or older than its sources."""
    from block_sparse_attention_bwd_b200 import _build

    _build.build()
