import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    # The tests load the in-tree library; build it (nvcc cross-compiles for
    # sm_100a without a GPU) when a fresh checkout has none yet.
    import __graft_entry__
    __graft_entry__._load_build_script().build()
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
