import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (runs on a B200)")


def pytest_sessionstart(session):
    # build the oracle and the CUDA library in-tree if they are missing or stale (nvcc
    # cross-compiles without a GPU)
    # (GQ_SKIP_CUDA_BUILD=1: runs of the oracle's pins alone, as the planted-mistake test does)
    from oracle import build as obuild
    obuild.build()
    if os.environ.get("GQ_SKIP_CUDA_BUILD") != "1":
        from gradient_quantization_communication_b200 import build as gbuild
        gbuild.build()
