import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libvsa")


def _stale(lib_path, src_dir):
    if not os.path.exists(lib_path):
        return True
    t = os.path.getmtime(lib_path)
    for d, _, files in os.walk(src_dir):
        for f in files:
            if os.path.getmtime(os.path.join(d, f)) > t:
                return True
    return os.path.getmtime(os.path.join(ROOT, "include", "vsa.h")) > t


@pytest.fixture(scope="session")
def libvsa():
    """The built C-ABI library (built in-tree first if missing or stale)."""
    from tile_sparse_video_b200 import build, vsa
    if _stale(build.LIB, build.CSRC):
        build.build()
    return vsa.lib()
