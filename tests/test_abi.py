"""The C-ABI library on the host (no GPU needed): it loads, exports every
entry point ``include/vsa.h`` declares, and its host planner reproduces the
oracle's tables bit for bit.  No kernel is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
from tile_sparse_video_b200 import vsa
from tile_sparse_video_b200.inputs import REF2VA, SMALL, TINY, VEDA_104K, sweep_workloads

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "vsa.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vsa_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(libvsa):
    decl = declared_symbols()
    assert len(decl) == 33
    assert sorted(vsa.EXPORTS) == decl
    for name in decl:
        assert hasattr(libvsa, name), name


GEOMS = [((40, 70), (4, 8, 8), (4, 4, 4)),
         ((5, 0, 64, 65), (5, 6, 7), (4, 4, 4)),
         ((), (4, 4, 4), (4, 4, 4)),
         ((130,), (0, 4, 4), (4, 4, 4)),
         ((256, 3), (8, 17, 9), (4, 8, 4)),
         ((1, 1, 1), (3, 3, 3), (4, 4, 4)),
         ((150, 1008, 414), (37, 24, 42), (4, 4, 4))]
GEOMS += [(w.prefix, w.grid, w.tile) for w in (TINY, SMALL, REF2VA, VEDA_104K)]
GEOMS += [(w.prefix, w.grid, w.tile) for w in sweep_workloads()[::5]]


@pytest.mark.parametrize("prefix,grid,tile", GEOMS)
def test_host_plan_matches_oracle(libvsa, prefix, grid, tile):
    p = vsa.Plan(prefix, grid, tile, device=-1)
    o = O.plan(prefix, grid, tile)
    assert (p.n_tokens, p.n_padded, p.n_tiles, p.n_prefix_tiles, p.tile_rows) == \
           (o.n_tokens, o.n_padded, o.n_tiles, o.n_prefix_tiles, o.R)
    t = p.tables()
    assert np.array_equal(t["untile"], o.untile)
    assert np.array_equal(t["row_src"], o.row_src)
    assert np.array_equal(t["block_len"], o.block_len)
    assert np.array_equal(t["tile_seg"], o.tile_seg)
    for ratio in (0.0, 0.05, 0.1, 0.25, 0.5, 1 - 0.95, 1.0):
        try:
            want = O.keep_count(o.n_video_tiles, o.n_prefix_tiles, keep_ratio=ratio)
        except ValueError:
            with pytest.raises(vsa.VsaError):
                p.keep_count(keep_ratio=ratio)
            continue
        assert p.keep_count(keep_ratio=ratio) == want
    for kt in (0, 1, 24, 10 ** 6):
        try:
            want = O.keep_count(o.n_video_tiles, o.n_prefix_tiles, keep_tiles=kt)
        except ValueError:
            with pytest.raises(vsa.VsaError):
                p.keep_count(keep_tiles=kt)
            continue
        assert p.keep_count(keep_tiles=kt) == want
    p.close()


def test_plan_errors(libvsa):
    with pytest.raises(vsa.VsaError) as e:
        vsa.Plan((10,), (4, 4, 4), (2, 2, 2), device=-1)          # R = 8
    assert e.value.status == 2
    with pytest.raises(vsa.VsaError) as e:
        vsa.Plan((10,), (-1, 4, 4), (4, 4, 4), device=-1)
    assert e.value.status == 3
    with pytest.raises(vsa.VsaError) as e:
        vsa.Plan((-3,), (4, 4, 4), (4, 4, 4), device=-1)
    assert e.value.status == 3


def test_host_only_plan_refuses_launches(libvsa):
    p = vsa.Plan((40, 70), (4, 8, 8), (4, 4, 4), device=-1)
    buf = (ctypes.c_uint8 * 64)()
    st = libvsa.vsa_permute(p.handle, ctypes.cast(buf, ctypes.c_void_p), ctypes.cast(buf, ctypes.c_void_p),
                            1, 2, 64, None)
    assert st == 1
    assert b"host-only" in libvsa.vsa_last_error()
    n = ctypes.c_size_t()
    assert libvsa.vsa_workspace_size(p.handle, 1, 2, 64, 2, ctypes.byref(n)) == 0
    # the pooled means, then the coarse kernel's score rows: 32 rows of
    # ceil4(T) floats for each of its 2 x 148 CTAs (a host-only plan assumes
    # 148 SMs)
    assert n.value == 3 * 1 * 2 * p.n_tiles * 64 * 4 + 2 * 148 * 32 * ((p.n_tiles + 3) // 4 * 4) * 4
    assert libvsa.vsa_workspace_size(p.handle, 1, 2, 96, 2, ctypes.byref(n)) == 2
    # the calls added for training and tile-before-projecting refuse a host-only plan too
    vp = ctypes.cast(buf, ctypes.c_void_p)
    assert libvsa.vsa_permute_rows(p.handle, vp, vp, 1, 64, None) == 1
    assert libvsa.vsa_project_tiled(p.handle, vp, vp, 1, 2, 64, 64, 0, vp, None) == 1
    assert libvsa.vsa_combine_backward(p.handle, vp, vp, vp, vp, 1, 2, 64, vp, vp, vp, None) == 1
    assert libvsa.vsa_check_bounded_wait(p.handle, vp, None) == 1
    assert b"host-only" in libvsa.vsa_last_error()
    # backward workspace: the larger of the coarse backward's P and dS (2 x [B*H, T, T]
    # fp32) and the attention backward's bitmap (B*H*T*ceil(T/32) words, 16-byte
    # rounded) plus its two work counters (16 bytes)
    assert libvsa.vsa_backward_workspace_size(p.handle, 1, 2, 64, ctypes.byref(n)) == 0
    T = p.n_tiles
    bitmap = (2 * T * ((T + 31) // 32) * 4 + 15) // 16 * 16 + 16
    assert n.value == max(2 * 2 * T * T * 4, bitmap)
    assert libvsa.vsa_backward_workspace_size(p.handle, 1, 2, 96, ctypes.byref(n)) == 2
    assert libvsa.vsa_plan_destroy(None) == 0
    p.close()


def test_runner_argument_checks(libvsa):
    """The host-buffer runner refuses what it cannot run before touching a
    device: NULL handles and host-only plans."""
    p = vsa.Plan((40, 70), (4, 8, 8), (4, 4, 4), device=-1)
    r = ctypes.c_void_p(1234)
    assert libvsa.vsa_runner_create(p.handle, 1, 2, 64, 2, 0.125, ctypes.byref(r)) == 1
    assert b"host-only" in libvsa.vsa_last_error()
    assert r.value is None                                       # *out cleared on failure
    assert libvsa.vsa_runner_create(None, 1, 2, 64, 2, 0.125, ctypes.byref(r)) == 1
    assert libvsa.vsa_runner_run(None, 1, None, None, None, None, None, None) == 1
    ms = ctypes.c_float()
    assert libvsa.vsa_runner_elapsed(None, ctypes.byref(ms)) == 1
    assert libvsa.vsa_runner_destroy(None) == 0
    p.close()
