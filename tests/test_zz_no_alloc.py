"""The allocation-free coarse/top-k entry point, called through the C ABI.

Callers that cannot call cudaMalloc (a host that owns all device memory and
gives plugins no allocator, or a loop that cannot afford cudaMalloc's implicit
device-wide synchronisation) use vsa_coarse_topk_noalloc, whose scratch lives
in a fixed array inside the library.  Its results must match the workspace
entry point's on two calls in a row (the second call finds the first call's
data still in the shared array), and sizes beyond the array are refused.

This file is named to be collected last, so a stop-at-first-failure run has
already run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests.parity import f64
from tile_sparse_video_b200 import vsa
from tile_sparse_video_b200.inputs import SMALL, VEDA_104K, make_inputs

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def test_noalloc_matches_workspace_entry_point(libvsa):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    w = SMALL
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    k = plan.keep_count(keep_ratio=w.keep_ratio)
    inp = make_inputs(w)
    q_t, k_t, v_t = (vsa.vsa_permute(plan, inp[x].cuda()) for x in "qkv")
    scale = w.D ** -0.5
    ref_oc, ref_idx, ref_s, _ = vsa.vsa_coarse_topk(plan, q_t, k_t, v_t, k, scale, want_scores=True)
    torch.cuda.synchronize()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        oc = torch.full_like(ref_oc, float("nan"))
        idx = torch.full_like(ref_idx, -1)
        sc = torch.full_like(ref_s, float("nan"))
        st = libvsa.vsa_coarse_topk_noalloc(plan.handle, _p(q_t), _p(k_t), _p(v_t), w.B, w.H, w.D,
                                            scale, k, _p(oc), _p(idx), _p(sc), stream)
        assert st == 0, libvsa.vsa_last_error()
        vsa.vsa_sync_status(plan)
        assert torch.equal(idx, ref_idx)
        np.testing.assert_allclose(f64(oc), f64(ref_oc), rtol=1e-4, atol=1e-5)
        np.testing.assert_allclose(f64(sc), f64(ref_s), rtol=1e-4, atol=1e-5)


def test_noalloc_refuses_sizes_beyond_its_array(libvsa):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    w = VEDA_104K                              # 3*42*818*128*4 bytes > 16 MiB
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    buf = torch.zeros(64, dtype=torch.float32, device="cuda")
    st = libvsa.vsa_coarse_topk_noalloc(plan.handle, _p(buf), _p(buf), _p(buf), 1, 42, 128, 0.1, 82,
                                        _p(buf), _p(buf), None, None)
    assert st == 4
    assert b"16777216" in libvsa.vsa_last_error()
    vsa.vsa_sync_status(plan)
