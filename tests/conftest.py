import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionstart(session):
    # libtern.so is a build product kept out of version control: build it when a
    # checkout has none (nvcc cross-compiles for sm_100a without a GPU). An
    # existing library is used as it is.
    if not os.path.exists(os.path.join(ROOT, "packed_ternary_weight_b200", "libtern.so")):
        from packed_ternary_weight_b200 import build
        build.build()
