import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_sessionstart(session):
    # the C-ABI library lives in-tree: build it (nvcc, sm_100a) if it is missing or older than
    # its sources, so that every test runs the current kernels; a failed build fails the session
    from sparse_moe_layer_03_b200 import build as B
    B.build()
