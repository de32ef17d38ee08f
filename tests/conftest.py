import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionstart(session):
    # The library is built in-tree (nvcc cross-compiles without a GPU); rebuild
    # only when a source is newer than libsbl.so.
    from sparse_linear_layers_b200.build import build_library
    build_library()
