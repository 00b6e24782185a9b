import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built library")


def pytest_sessionstart(session):
    # Build libqlinear.so in-tree if it is missing or older than its sources
    # (nvcc cross-compiles without a GPU).
    from trellis_coded_matmul_b200 import build
    build.build()
