import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built library")


def pytest_sessionstart(session):
    # Build libqlinear.so in-tree if it is missing or older than its sources
    # (nvcc cross-compiles without a GPU).  The build script is loaded by path
    # so that a stale library is never imported before it is rebuilt.
    path = os.path.join(ROOT, "trellis_coded_matmul_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_tcm_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
