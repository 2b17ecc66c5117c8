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


@pytest.fixture(autouse=True)
def _name_parity_records(request):
    from tests import parity
    parity.CURRENT_TEST[0] = request.node.name
    yield


def pytest_terminal_summary(terminalreporter):
    """Output comparisons against their bf16 floor: the error of the oracle
    itself rounded to bf16, next to the kernel's error."""
    from tests.parity import RECORDS
    if not RECORDS:
        return
    tr = terminalreporter
    tr.write_sep("-", "output error vs bf16 floor (max / mean)")
    worst_max = max(r[1] / r[3] for r in RECORDS if r[3] > 0)
    worst_mean = max(r[2] / r[4] for r in RECORDS if r[4] > 0)
    for what, mx, mn, fmx, fmn in RECORDS:
        tr.write_line(f"{what:70s} err {mx:.2e} / {mn:.2e}   floor {fmx:.2e} / {fmn:.2e}   "
                      f"ratio {mx / fmx if fmx else 0:.2f} / {mn / fmn if fmn else 0:.2f}")
    tr.write_line(f"largest ratios: max {worst_max:.2f}, mean {worst_mean:.2f} ({len(RECORDS)} comparisons)")
