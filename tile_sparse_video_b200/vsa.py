"""Thin Python binding of libvsa (ctypes).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is no
fallback: if ``libvsa.so`` is missing, every call raises.

The names mirror the C ABI in ``include/vsa.h``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvsa.so")
_lib = None

VSA_OK = 0
STATUS_NAMES = {0: "VSA_OK", 1: "VSA_ERR_INVALID_ARG", 2: "VSA_ERR_UNSUPPORTED", 3: "VSA_ERR_PLAN",
                4: "VSA_ERR_WORKSPACE", 5: "VSA_ERR_CUDA", 6: "VSA_ERR_DEVICE_TIMEOUT",
                7: "VSA_ERR_DEVICE_INDEX"}

# exported C symbols (kept in step with include/vsa.h)
EXPORTS = ("vsa_plan_create", "vsa_plan_info", "vsa_plan_tables", "vsa_keep_count",
           "vsa_plan_destroy", "vsa_workspace_size", "vsa_permute", "vsa_unpermute",
           "vsa_permute_pool", "vsa_coarse_topk", "vsa_coarse_topk_pooled",
           "vsa_coarse_topk_noalloc", "vsa_sparse_attn", "vsa_sparse_attn_combine",
           "vsa_gate_combine", "vsa_project", "vsa_project_tiled", "vsa_permute_rows",
           "vsa_keep_count_ref", "vsa_select_reference",
           "vsa_sparse_attn_ref", "vsa_backward_workspace_size", "vsa_combine_backward",
           "vsa_coarse_backward", "vsa_sparse_attn_backward", "vsa_check_bounded_wait",
           "vsa_runner_create", "vsa_runner_run", "vsa_runner_elapsed", "vsa_runner_destroy",
           "vsa_debug_set_wait_limit", "vsa_sync_status", "vsa_last_error")


class VsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class _Geometry(ctypes.Structure):
    _fields_ = [("n_prefix_segments", ctypes.c_int32), ("prefix_lens", ctypes.POINTER(ctypes.c_int64)),
                ("grid_t", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("tile_t", ctypes.c_int32), ("tile_h", ctypes.c_int32), ("tile_w", ctypes.c_int32)]


def lib():
    """Load libvsa.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m tile_sparse_video_b200.build` (no fallback exists)")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, I32, I64, F, D, Z, V = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int32, ctypes.c_int64,
                                      ctypes.c_float, ctypes.c_double, ctypes.c_size_t, ctypes.c_void_p)
        sig = {
            "vsa_plan_create": [ctypes.POINTER(_Geometry), I, ctypes.POINTER(P)],
            "vsa_plan_info": [P, ctypes.POINTER(I64), ctypes.POINTER(I64), ctypes.POINTER(I32),
                              ctypes.POINTER(I32), ctypes.POINTER(I32)],
            "vsa_plan_tables": [P, V, V, V, V],
            "vsa_keep_count": [P, D, I32, ctypes.POINTER(I32)],
            "vsa_plan_destroy": [P],
            "vsa_workspace_size": [P, I, I, I, I, ctypes.POINTER(Z)],
            "vsa_permute": [P, V, V, I, I, I, V],
            "vsa_unpermute": [P, V, V, I, I, I, V],
            "vsa_permute_pool": [P, V, V, I, I, I, V, V],
            "vsa_coarse_topk_pooled": [P, I, I, I, F, I, V, V, V, V, Z, V],
            "vsa_coarse_topk": [P, V, V, V, I, I, I, F, I, V, V, V, V, Z, V],
            "vsa_coarse_topk_noalloc": [P, V, V, V, I, I, I, F, I, V, V, V, V],
            "vsa_sparse_attn": [P, V, V, V, V, I, I, I, I, F, V, V, V, Z, V],
            "vsa_sparse_attn_combine": [P, V, V, V, V, I, I, I, I, F, V, V, V, V, V],
            "vsa_gate_combine": [P, V, V, V, V, I, I, I, I, V],
            "vsa_project": [P, V, V, I, I, I, I, I, V, V],
            "vsa_project_tiled": [P, V, V, I, I, I, I, I, V, V],
            "vsa_permute_rows": [P, V, V, I, I, V],
            "vsa_keep_count_ref": [P, D, I32, ctypes.POINTER(I32)],
            "vsa_select_reference": [P, I, I, I, F, I, V, V, Z, V],
            "vsa_sparse_attn_ref": [P, V, V, V, V, I, V, I, I, I, I, F, V, V, V, V, V],
            "vsa_backward_workspace_size": [P, I, I, I, ctypes.POINTER(Z)],
            "vsa_combine_backward": [P, V, V, V, V, I, I, I, V, V, V, V],
            "vsa_coarse_backward": [P, V, V, V, V, I, I, I, F, V, V, V, V, Z, V],
            "vsa_sparse_attn_backward": [P, V, V, V, V, V, I, V, I, V, V, V, V, V, I, I, I, F,
                                         V, V, V, V, Z, V],
            "vsa_check_bounded_wait": [P, V, V],
            "vsa_runner_create": [P, I, I, I, I, F, ctypes.POINTER(P)],
            "vsa_runner_run": [P, I, V, V, V, V, V, V],
            "vsa_runner_elapsed": [P, ctypes.POINTER(F)],
            "vsa_runner_destroy": [P],
            "vsa_debug_set_wait_limit": [ctypes.c_uint64],
            "vsa_sync_status": [P, V],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.vsa_last_error.argtypes = []
        L.vsa_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status: int):
    if status != VSA_OK:
        raise VsaError(status, lib().vsa_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class Plan:
    """Owner of a libvsa plan (step 1 tables).  ``device=-1`` builds a host-only
    plan (tables and keep counts, no launches)."""

    def __init__(self, prefix_lens: Sequence[int], grid: Sequence[int], tile: Sequence[int],
                 device: Optional[int] = None):
        L = lib()
        if device is None:
            device = torch.cuda.current_device()
        self.prefix_lens = tuple(int(x) for x in prefix_lens)
        self.grid, self.tile = tuple(int(x) for x in grid), tuple(int(x) for x in tile)
        self._lens = (ctypes.c_int64 * max(1, len(self.prefix_lens)))(*self.prefix_lens)
        geo = _Geometry(len(self.prefix_lens), ctypes.cast(self._lens, ctypes.POINTER(ctypes.c_int64)),
                        *self.grid, *self.tile)
        h = ctypes.c_void_p()
        _check(L.vsa_plan_create(ctypes.byref(geo), int(device), ctypes.byref(h)))
        self._h = h
        self.device = int(device)
        n_tok, n_pad = ctypes.c_int64(), ctypes.c_int64()
        T, n_p, R = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        _check(L.vsa_plan_info(h, ctypes.byref(n_tok), ctypes.byref(n_pad), ctypes.byref(T),
                               ctypes.byref(n_p), ctypes.byref(R)))
        self.n_tokens, self.n_padded = n_tok.value, n_pad.value
        self.n_tiles, self.n_prefix_tiles, self.tile_rows = T.value, n_p.value, R.value
        self.n_video_tiles = self.n_tiles - self.n_prefix_tiles

    @property
    def handle(self):
        return self._h

    def tables(self) -> dict:
        out = {"untile": np.empty(self.n_tokens, np.int32), "row_src": np.empty(self.n_padded, np.int32),
               "block_len": np.empty(self.n_tiles, np.int32), "tile_seg": np.empty(self.n_tiles, np.int32)}
        _check(lib().vsa_plan_tables(self._h, *(ctypes.c_void_p(a.ctypes.data) for a in out.values())))
        return out

    def keep_count(self, keep_ratio: Optional[float] = None, keep_tiles: Optional[int] = None) -> int:
        k = ctypes.c_int32()
        _check(lib().vsa_keep_count(self._h, float(keep_ratio if keep_ratio is not None else 0.0),
                                    int(keep_tiles) if keep_tiles is not None else -1, ctypes.byref(k)))
        return k.value

    def workspace_size(self, B: int, H: int, D: int, k: int) -> int:
        n = ctypes.c_size_t()
        _check(lib().vsa_workspace_size(self._h, B, H, D, k, ctypes.byref(n)))
        return n.value

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().vsa_plan_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def vsa_plan(prefix_lens, grid, tile, device=None) -> Plan:
    return Plan(prefix_lens, grid, tile, device)


def vsa_permute(plan: Plan, x: torch.Tensor, x_t: Optional[torch.Tensor] = None, stream=None):
    B, H, N, D = x.shape
    _need(x, "x", torch.bfloat16, (B, H, plan.n_tokens, D))
    if x_t is None:
        x_t = torch.empty(B, H, plan.n_padded, D, dtype=torch.bfloat16, device=x.device)
    _need(x_t, "x_t", torch.bfloat16, (B, H, plan.n_padded, D))
    _check(lib().vsa_permute(plan.handle, _ptr(x), _ptr(x_t), B, H, D, _stream(stream)))
    return x_t


def vsa_unpermute(plan: Plan, x_t: torch.Tensor, x: Optional[torch.Tensor] = None, stream=None):
    B, H, _, D = x_t.shape
    _need(x_t, "x_t", torch.bfloat16, (B, H, plan.n_padded, D))
    if x is None:
        x = torch.empty(B, H, plan.n_tokens, D, dtype=torch.bfloat16, device=x_t.device)
    _need(x, "x", torch.bfloat16, (B, H, plan.n_tokens, D))
    _check(lib().vsa_unpermute(plan.handle, _ptr(x_t), _ptr(x), B, H, D, _stream(stream)))
    return x


def vsa_coarse_topk(plan: Plan, q_t, k_t, v_t, k: int, scale: Optional[float] = None, ws=None,
                    o_coarse=None, topk_idx=None, want_scores: bool = False, stream=None):
    """Returns (o_coarse fp32 [B,H,T,D], topk_idx int32 [B,H,n_v,k], scores or None, ws)."""
    B, H, _, D = q_t.shape
    for name, t in (("q_t", q_t), ("k_t", k_t), ("v_t", v_t)):
        _need(t, name, torch.bfloat16, (B, H, plan.n_padded, D))
    dev = q_t.device
    scale = D ** -0.5 if scale is None else float(scale)
    T, n_v = plan.n_tiles, plan.n_video_tiles
    if o_coarse is None:
        o_coarse = torch.empty(B, H, T, D, dtype=torch.float32, device=dev)
    if topk_idx is None:
        topk_idx = torch.empty(B, H, n_v, max(k, 0), dtype=torch.int32, device=dev)
    scores = torch.empty(B, H, n_v, max(k, 0), dtype=torch.float32, device=dev) if want_scores else None
    need = plan.workspace_size(B, H, D, k)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().vsa_coarse_topk(plan.handle, _ptr(q_t), _ptr(k_t), _ptr(v_t), B, H, D, scale, k,
                                 _ptr(o_coarse), _ptr(topk_idx) if topk_idx.numel() else None,
                                 _ptr(scores) if scores is not None and scores.numel() else None,
                                 _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    return o_coarse, topk_idx, scores, ws


def vsa_permute_pool(plan: Plan, x: torch.Tensor, x_t: Optional[torch.Tensor] = None,
                     pooled: Optional[torch.Tensor] = None, stream=None):
    """Permute x into x_t and write the fp32 per-tile means of its live rows to
    pooled [B,H,T,D] in the same pass.  Returns (x_t, pooled)."""
    B, H, N, D = x.shape
    _need(x, "x", torch.bfloat16, (B, H, plan.n_tokens, D))
    if x_t is None:
        x_t = torch.empty(B, H, plan.n_padded, D, dtype=torch.bfloat16, device=x.device)
    _need(x_t, "x_t", torch.bfloat16, (B, H, plan.n_padded, D))
    if pooled is None:
        pooled = torch.empty(B, H, plan.n_tiles, D, dtype=torch.float32, device=x.device)
    _need(pooled, "pooled", torch.float32, (B, H, plan.n_tiles, D))
    _check(lib().vsa_permute_pool(plan.handle, _ptr(x), _ptr(x_t), B, H, D, _ptr(pooled),
                                  _stream(stream)))
    return x_t, pooled


def pooled_slots(plan: Plan, ws: torch.Tensor, B: int, H: int, D: int):
    """Views of the workspace's qbar, kbar, vbar slots (fp32 [B,H,T,D] each)."""
    n = B * H * plan.n_tiles * D
    f = ws[: 3 * n * 4].view(torch.float32)
    return tuple(f[i * n:(i + 1) * n].view(B, H, plan.n_tiles, D) for i in range(3))


def vsa_coarse_topk_pooled(plan: Plan, B: int, H: int, D: int, k: int, ws, scale: Optional[float] = None,
                           o_coarse=None, topk_idx=None, want_scores: bool = False, stream=None):
    """vsa_coarse_topk from pooled means already in ``ws`` (written by
    vsa_permute_pool into pooled_slots(ws)).  Returns (o_coarse, topk_idx,
    scores or None)."""
    dev = ws.device
    scale = D ** -0.5 if scale is None else float(scale)
    T, n_v = plan.n_tiles, plan.n_video_tiles
    if o_coarse is None:
        o_coarse = torch.empty(B, H, T, D, dtype=torch.float32, device=dev)
    if topk_idx is None:
        topk_idx = torch.empty(B, H, n_v, max(k, 0), dtype=torch.int32, device=dev)
    scores = torch.empty(B, H, n_v, max(k, 0), dtype=torch.float32, device=dev) if want_scores else None
    _check(lib().vsa_coarse_topk_pooled(plan.handle, B, H, D, scale, k, _ptr(o_coarse),
                                        _ptr(topk_idx) if topk_idx.numel() else None,
                                        _ptr(scores) if scores is not None and scores.numel() else None,
                                        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    return o_coarse, topk_idx, scores


def vsa_coarse_topk_noalloc(plan: Plan, q_t, k_t, v_t, k: int, scale: Optional[float] = None,
                            o_coarse=None, topk_idx=None, want_scores: bool = False, stream=None):
    """Like vsa_coarse_topk, but the library keeps the scratch in its own fixed
    16 MiB device array (for callers that cannot allocate).  Returns
    (o_coarse, topk_idx, scores or None)."""
    B, H, _, D = q_t.shape
    for name, t in (("q_t", q_t), ("k_t", k_t), ("v_t", v_t)):
        _need(t, name, torch.bfloat16, (B, H, plan.n_padded, D))
    dev = q_t.device
    scale = D ** -0.5 if scale is None else float(scale)
    if o_coarse is None:
        o_coarse = torch.empty(B, H, plan.n_tiles, D, dtype=torch.float32, device=dev)
    if topk_idx is None:
        topk_idx = torch.empty(B, H, plan.n_video_tiles, max(k, 0), dtype=torch.int32, device=dev)
    scores = (torch.empty(B, H, plan.n_video_tiles, max(k, 0), dtype=torch.float32, device=dev)
              if want_scores else None)
    _check(lib().vsa_coarse_topk_noalloc(plan.handle, _ptr(q_t), _ptr(k_t), _ptr(v_t), B, H, D, scale,
                                         k, _ptr(o_coarse), _ptr(topk_idx) if topk_idx.numel() else None,
                                         _ptr(scores) if scores is not None and scores.numel() else None,
                                         _stream(stream)))
    return o_coarse, topk_idx, scores


def vsa_sparse_attn(plan: Plan, q_t, k_t, v_t, topk_idx, k: int, scale: Optional[float] = None,
                    out=None, want_lse: bool = False, stream=None):
    """Returns (o_fine_t bf16 [B,H,N_pad,D], lse fp32 [B,H,N_pad] or None)."""
    B, H, _, D = q_t.shape
    for name, t in (("q_t", q_t), ("k_t", k_t), ("v_t", v_t)):
        _need(t, name, torch.bfloat16, (B, H, plan.n_padded, D))
    _need(topk_idx, "topk_idx", torch.int32, (B, H, plan.n_video_tiles, max(k, 0)))
    scale = D ** -0.5 if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q_t)
    lse = torch.empty(B, H, plan.n_padded, dtype=torch.float32, device=q_t.device) if want_lse else None
    _check(lib().vsa_sparse_attn(plan.handle, _ptr(q_t), _ptr(k_t), _ptr(v_t),
                                 _ptr(topk_idx) if topk_idx.numel() else None, B, H, D, k, scale,
                                 _ptr(out), _ptr(lse), None, 0, _stream(stream)))
    return out, lse


def vsa_sparse_attn_combine(plan: Plan, q_t, k_t, v_t, topk_idx, k: int, gate, o_coarse,
                            scale: Optional[float] = None, out=None, want_lse: bool = False,
                            stream=None):
    """Attention with the gated combine fused into its epilogue; ``gate`` is in
    natural order.  Returns (out bf16 [B,H,N,D] natural order, lse or None)."""
    B, H, _, D = q_t.shape
    for name, t in (("q_t", q_t), ("k_t", k_t), ("v_t", v_t)):
        _need(t, name, torch.bfloat16, (B, H, plan.n_padded, D))
    _need(topk_idx, "topk_idx", torch.int32, (B, H, plan.n_video_tiles, max(k, 0)))
    _need(gate, "gate", torch.bfloat16, (B, H, plan.n_tokens, D))
    _need(o_coarse, "o_coarse", torch.float32, (B, H, plan.n_tiles, D))
    scale = D ** -0.5 if scale is None else float(scale)
    if out is None:
        out = torch.empty(B, H, plan.n_tokens, D, dtype=torch.bfloat16, device=q_t.device)
    _need(out, "out", torch.bfloat16, (B, H, plan.n_tokens, D))
    lse = torch.empty(B, H, plan.n_padded, dtype=torch.float32, device=q_t.device) if want_lse else None
    _check(lib().vsa_sparse_attn_combine(plan.handle, _ptr(q_t), _ptr(k_t), _ptr(v_t),
                                         _ptr(topk_idx) if topk_idx.numel() else None, B, H, D, k,
                                         scale, _ptr(gate), _ptr(o_coarse), _ptr(out), _ptr(lse),
                                         _stream(stream)))
    return out, lse


def vsa_gate_combine(plan: Plan, o_fine_t, gate_t, o_coarse, natural: bool = True, out=None,
                     stream=None):
    B, H, _, D = o_fine_t.shape
    _need(o_fine_t, "o_fine_t", torch.bfloat16, (B, H, plan.n_padded, D))
    _need(gate_t, "gate_t", torch.bfloat16, (B, H, plan.n_padded, D))
    _need(o_coarse, "o_coarse", torch.float32, (B, H, plan.n_tiles, D))
    rows = plan.n_tokens if natural else plan.n_padded
    if out is None:
        out = torch.empty(B, H, rows, D, dtype=torch.bfloat16, device=o_fine_t.device)
    _need(out, "out", torch.bfloat16, (B, H, rows, D))
    _check(lib().vsa_gate_combine(plan.handle, _ptr(o_fine_t), _ptr(gate_t), _ptr(o_coarse), _ptr(out),
                                  1 if natural else 0, B, H, D, _stream(stream)))
    return out


def vsa_project(plan: Plan, x: torch.Tensor, w: torch.Tensor, H: int, D: int, sigmoid: bool = False,
                y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y[b,h,n,d] = act(sum_c x[b,n,c] w[h*D+d,c]) (tcgen05 GEMM; act = sigmoid or
    identity).  x bf16 [B,N,C], w bf16 [H*D,C]; returns y bf16 [B,H,N,D]."""
    B, N, C = x.shape
    _need(x, "x", torch.bfloat16, (B, plan.n_tokens, C))
    _need(w, "w", torch.bfloat16, (H * D, C))
    if y is None:
        y = torch.empty(B, H, plan.n_tokens, D, dtype=torch.bfloat16, device=x.device)
    _need(y, "y", torch.bfloat16, (B, H, plan.n_tokens, D))
    _check(lib().vsa_project(plan.handle, _ptr(x), _ptr(w), B, H, D, C, 1 if sigmoid else 0, _ptr(y),
                             _stream(stream)))
    return y


def vsa_permute_rows(plan: Plan, x: torch.Tensor, x_t: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Tile order for rows of any width: x bf16 [B,N,C] -> x_t bf16 [B,N_pad,C]
    (pad rows 0), the layer input before its projections."""
    B, N, C = x.shape
    _need(x, "x", torch.bfloat16, (B, plan.n_tokens, C))
    if x_t is None:
        x_t = torch.empty(B, plan.n_padded, C, dtype=torch.bfloat16, device=x.device)
    _need(x_t, "x_t", torch.bfloat16, (B, plan.n_padded, C))
    _check(lib().vsa_permute_rows(plan.handle, _ptr(x), _ptr(x_t), B, C, _stream(stream)))
    return x_t


def vsa_project_tiled(plan: Plan, x_t: torch.Tensor, w: torch.Tensor, H: int, D: int,
                      sigmoid: bool = False, y_t: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """vsa_project on tiled rows: x_t bf16 [B,N_pad,C] (from vsa_permute_rows),
    w bf16 [H*D,C]; returns y_t bf16 [B,H,N_pad,D] in tile order."""
    B, Np, C = x_t.shape
    _need(x_t, "x_t", torch.bfloat16, (B, plan.n_padded, C))
    _need(w, "w", torch.bfloat16, (H * D, C))
    if y_t is None:
        y_t = torch.empty(B, H, plan.n_padded, D, dtype=torch.bfloat16, device=x_t.device)
    _need(y_t, "y_t", torch.bfloat16, (B, H, plan.n_padded, D))
    _check(lib().vsa_project_tiled(plan.handle, _ptr(x_t), _ptr(w), B, H, D, C, 1 if sigmoid else 0,
                                   _ptr(y_t), _stream(stream)))
    return y_t


class TiledInputProjection:
    """Q, K, V and the gate of a layer from its input x [B,N,C], tiled before
    projecting: one vsa_permute_rows of x, then four tcgen05 GEMMs on the tiled
    rows (vsa_project_tiled) writing q_t, k_t, v_t and g_t [B,H,N_pad,D] in tile
    order, ready for vsa_coarse_topk, vsa_sparse_attn and vsa_gate_combine.
    Weights are nn.Linear layout [H*D, C], bias-free."""

    def __init__(self, plan: Plan, B: int, H: int, D: int, C: int, device=None):
        self.plan, self.B, self.H, self.D, self.C = plan, B, H, D, C
        dev = torch.device("cuda", plan.device) if device is None else torch.device(device)
        self.x_t = torch.empty(B, plan.n_padded, C, dtype=torch.bfloat16, device=dev)
        self.out = tuple(torch.empty(B, H, plan.n_padded, D, dtype=torch.bfloat16, device=dev)
                         for _ in range(4))

    def __call__(self, x, w_q, w_k, w_v, w_g, stream=None):
        p = self.plan
        vsa_permute_rows(p, x, self.x_t, stream)
        for w, y in zip((w_q, w_k, w_v, w_g), self.out):
            vsa_project_tiled(p, self.x_t, w, self.H, self.D, y_t=y, stream=stream)
        return self.out


def vsa_keep_count_ref(plan: Plan, keep_ratio: Optional[float] = None,
                       keep_tiles: Optional[int] = None) -> int:
    """Reference tiles each video query tile keeps (reference_sparsity)."""
    out = ctypes.c_int32()
    _check(lib().vsa_keep_count_ref(plan.handle, 0.0 if keep_ratio is None else float(keep_ratio),
                                    -1 if keep_tiles is None else int(keep_tiles), ctypes.byref(out)))
    return out.value


def vsa_select_reference(plan: Plan, B: int, H: int, D: int, k_ref: int, ws,
                         scale: Optional[float] = None, out=None, stream=None):
    """Top k_ref reference tiles of every video query tile from the pooled
    means in ``ws``; returns int32 [B,H,n_v,k_ref]."""
    scale = D ** -0.5 if scale is None else float(scale)
    if out is None:
        out = torch.empty(B, H, plan.n_video_tiles, max(k_ref, 0), dtype=torch.int32, device=ws.device)
    _check(lib().vsa_select_reference(plan.handle, B, H, D, scale, k_ref,
                                      _ptr(out) if out.numel() else None, _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)))
    return out


def vsa_sparse_attn_ref(plan: Plan, q_t, k_t, v_t, topk_idx, k: int, topk_ref, k_ref: int,
                        scale: Optional[float] = None, gate=None, o_coarse=None, out=None,
                        want_lse: bool = False, stream=None):
    """Sparse attention with the video query tiles' reference tiles thinned to
    ``topk_ref``.  gate/o_coarse given: fused combine, natural-order output;
    else o_fine in the padded layout.  Returns (out, lse or None)."""
    B, H, _, D = q_t.shape
    scale = D ** -0.5 if scale is None else float(scale)
    dev = q_t.device
    fused = gate is not None
    if out is None:
        rows = plan.n_tokens if fused else plan.n_padded
        out = torch.empty(B, H, rows, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, plan.n_padded, dtype=torch.float32, device=dev) if want_lse else None
    _check(lib().vsa_sparse_attn_ref(plan.handle, _ptr(q_t), _ptr(k_t), _ptr(v_t),
                                     _ptr(topk_idx) if topk_idx is not None and topk_idx.numel() else None, k,
                                     _ptr(topk_ref) if topk_ref is not None and topk_ref.numel() else None, k_ref,
                                     B, H, D, scale, _ptr(gate) if fused else None,
                                     _ptr(o_coarse) if fused else None, _ptr(out), _ptr(lse),
                                     _stream(stream)))
    return out, lse


def vsa_debug_set_wait_limit(ns: int) -> None:
    """Bound of the attention kernels' mbarrier waits from now on, in ns
    (0: the 2 s default).  A test hook for the kernels' abort path."""
    _check(lib().vsa_debug_set_wait_limit(int(ns)))


def vsa_sync_status(plan: Plan, stream=None):
    _check(lib().vsa_sync_status(plan.handle, _stream(stream)))


def vsa_check_bounded_wait(plan: Plan, stream=None) -> torch.Tensor:
    """Launch the bounded-wait self-test (its waits give up after 2 s); returns
    the device int32[2] result (0 = that wait gave up).  Read the recorded
    timeout with vsa_sync_status, which raises VsaError(VSA_ERR_DEVICE_TIMEOUT)."""
    result = torch.full((4,), -1, dtype=torch.int32, device=torch.device("cuda", plan.device))
    _check(lib().vsa_check_bounded_wait(plan.handle, _ptr(result), _stream(stream)))
    return result[:2]


# ---------------------------------------------------------------- backward

def vsa_backward_workspace_size(plan: Plan, B: int, H: int, D: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().vsa_backward_workspace_size(plan.handle, B, H, D, ctypes.byref(n)))
    return int(n.value)


def vsa_combine_backward(plan: Plan, d_out_t, o_fine_t, gate_t, o_coarse, delta=None, d_gate_t=None,
                         d_o_coarse=None, stream=None):
    """Backward of the gated combine.  Returns (delta fp32 [B,H,N_pad],
    d_gate_t bf16 [B,H,N_pad,D], d_o_coarse fp32 [B,H,T,D])."""
    B, H, _, D = d_out_t.shape
    tiled = (B, H, plan.n_padded, D)
    for name, t in (("d_out_t", d_out_t), ("o_fine_t", o_fine_t), ("gate_t", gate_t)):
        _need(t, name, torch.bfloat16, tiled)
    _need(o_coarse, "o_coarse", torch.float32, (B, H, plan.n_tiles, D))
    dev = d_out_t.device
    if delta is None:
        delta = torch.empty(B, H, plan.n_padded, dtype=torch.float32, device=dev)
    if d_gate_t is None:
        d_gate_t = torch.empty(tiled, dtype=torch.bfloat16, device=dev)
    if d_o_coarse is None:
        d_o_coarse = torch.empty(B, H, plan.n_tiles, D, dtype=torch.float32, device=dev)
    _check(lib().vsa_combine_backward(plan.handle, _ptr(d_out_t), _ptr(o_fine_t), _ptr(gate_t),
                                      _ptr(o_coarse), B, H, D, _ptr(delta), _ptr(d_gate_t),
                                      _ptr(d_o_coarse), _stream(stream)))
    return delta, d_gate_t, d_o_coarse


def vsa_coarse_backward(plan: Plan, qbar, kbar, vbar, d_o_coarse, ws, scale: Optional[float] = None,
                        out=None, stream=None):
    """Backward of the coarse attention: (d_qbar, d_kbar, d_vbar), fp32 [B,H,T,D]."""
    B, H, T, D = qbar.shape
    for name, t in (("qbar", qbar), ("kbar", kbar), ("vbar", vbar), ("d_o_coarse", d_o_coarse)):
        _need(t, name, torch.float32, (B, H, plan.n_tiles, D))
    scale = D ** -0.5 if scale is None else float(scale)
    if out is None:
        out = tuple(torch.empty_like(qbar) for _ in range(3))
    _check(lib().vsa_coarse_backward(plan.handle, _ptr(qbar), _ptr(kbar), _ptr(vbar),
                                     _ptr(d_o_coarse), B, H, D, scale, _ptr(out[0]), _ptr(out[1]),
                                     _ptr(out[2]), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream(stream)))
    return out


def vsa_sparse_attn_backward(plan: Plan, q_t, k_t, v_t, d_out_t, topk_idx, k: int, lse, delta, ws,
                             topk_ref=None, k_ref: Optional[int] = None, d_bar=None,
                             scale: Optional[float] = None, out=None, stream=None):
    """Backward of the block-sparse attention (plus the pooling term when
    ``d_bar`` = (d_qbar, d_kbar, d_vbar) is given).  k_ref None: every
    reference tile is a key of every video query tile.  Returns (dq_t, dk_t,
    dv_t), bf16 [B,H,N_pad,D]."""
    B, H, _, D = q_t.shape
    tiled = (B, H, plan.n_padded, D)
    for name, t in (("q_t", q_t), ("k_t", k_t), ("v_t", v_t), ("d_out_t", d_out_t)):
        _need(t, name, torch.bfloat16, tiled)
    _need(lse, "lse", torch.float32, (B, H, plan.n_padded))
    _need(delta, "delta", torch.float32, (B, H, plan.n_padded))
    scale = D ** -0.5 if scale is None else float(scale)
    if out is None:
        out = tuple(torch.empty(tiled, dtype=torch.bfloat16, device=q_t.device) for _ in range(3))
    kr = plan.n_prefix_tiles if k_ref is None else int(k_ref)
    ref = None if k_ref is None or topk_ref is None or topk_ref.numel() == 0 else _ptr(topk_ref)
    db = (None, None, None) if d_bar is None else tuple(_ptr(t) for t in d_bar)
    _check(lib().vsa_sparse_attn_backward(
        plan.handle, _ptr(q_t), _ptr(k_t), _ptr(v_t), _ptr(d_out_t),
        _ptr(topk_idx) if topk_idx is not None and topk_idx.numel() else None, k, ref, kr,
        _ptr(lse), _ptr(delta), db[0], db[1], db[2], B, H, D, scale, _ptr(out[0]), _ptr(out[1]),
        _ptr(out[2]), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    return out


class Layer:
    """The five steps in sequence on caller-visible buffers, all launches on
    one stream.  ``fused=True`` (default): permute Q, K, V with the tile means
    taken in the same pass; coarse + top-k from those means; attention with
    the gated combine fused into its epilogue, writing natural order (the gate
    is read in natural order): 5 launches.  ``fused=False``: the unfused chain
    (permute Q, K, V, G; pool + coarse + top-k; attention; combine).  Buffers
    are allocated once and reused by every call."""

    def __init__(self, plan: Plan, B: int, H: int, D: int, k: int, scale: Optional[float] = None,
                 device=None, fused: bool = True, k_ref: Optional[int] = None):
        self.plan, self.B, self.H, self.D, self.k, self.fused = plan, B, H, D, k, fused
        # k_ref: reference tiles each video query tile keeps (None: all of them)
        self.k_ref = k_ref
        self.scale = D ** -0.5 if scale is None else float(scale)
        dev = torch.device("cuda", plan.device) if device is None else torch.device(device)
        tiled = (B, H, plan.n_padded, D)
        self.q_t, self.k_t, self.v_t = (torch.empty(tiled, dtype=torch.bfloat16, device=dev)
                                        for _ in range(3))
        self.g_t = None if fused else torch.empty(tiled, dtype=torch.bfloat16, device=dev)
        self.o_fine_t = None if fused else torch.empty(tiled, dtype=torch.bfloat16, device=dev)
        self.o_coarse = torch.empty(B, H, plan.n_tiles, D, dtype=torch.float32, device=dev)
        self.topk_idx = torch.empty(B, H, plan.n_video_tiles, max(k, 0), dtype=torch.int32, device=dev)
        self.ws = torch.empty(max(plan.workspace_size(B, H, D, k), 16), dtype=torch.uint8, device=dev)
        self.out = torch.empty(B, H, plan.n_tokens, D, dtype=torch.bfloat16, device=dev)
        self.topk_ref = (torch.empty(B, H, plan.n_video_tiles, max(k_ref, 0), dtype=torch.int32, device=dev)
                         if k_ref is not None else None)

    def __call__(self, q, k, v, g, stream=None):
        p = self.plan
        if self.fused:
            qbar, kbar, vbar = pooled_slots(p, self.ws, self.B, self.H, self.D)
            vsa_permute_pool(p, q, self.q_t, qbar, stream)
            vsa_permute_pool(p, k, self.k_t, kbar, stream)
            vsa_permute_pool(p, v, self.v_t, vbar, stream)
            vsa_coarse_topk_pooled(p, self.B, self.H, self.D, self.k, self.ws, self.scale,
                                   o_coarse=self.o_coarse, topk_idx=self.topk_idx, stream=stream)
            if self.k_ref is not None:
                vsa_select_reference(p, self.B, self.H, self.D, self.k_ref, self.ws, self.scale,
                                     out=self.topk_ref, stream=stream)
                vsa_sparse_attn_ref(p, self.q_t, self.k_t, self.v_t, self.topk_idx, self.k,
                                    self.topk_ref, self.k_ref, self.scale, gate=g,
                                    o_coarse=self.o_coarse, out=self.out, stream=stream)
                return self.out
            vsa_sparse_attn_combine(p, self.q_t, self.k_t, self.v_t, self.topk_idx, self.k, g,
                                    self.o_coarse, self.scale, out=self.out, stream=stream)
            return self.out
        vsa_permute(p, q, self.q_t, stream)
        vsa_permute(p, k, self.k_t, stream)
        vsa_permute(p, v, self.v_t, stream)
        vsa_coarse_topk(p, self.q_t, self.k_t, self.v_t, self.k, self.scale, ws=self.ws,
                        o_coarse=self.o_coarse, topk_idx=self.topk_idx, stream=stream)
        vsa_permute(p, g, self.g_t, stream)
        if self.k_ref is not None:
            vsa_select_reference(p, self.B, self.H, self.D, self.k_ref, self.ws, self.scale,
                                 out=self.topk_ref, stream=stream)
            vsa_sparse_attn_ref(p, self.q_t, self.k_t, self.v_t, self.topk_idx, self.k,
                                self.topk_ref, self.k_ref, self.scale, out=self.o_fine_t, stream=stream)
        else:
            vsa_sparse_attn(p, self.q_t, self.k_t, self.v_t, self.topk_idx, self.k, self.scale,
                            out=self.o_fine_t, stream=stream)
        vsa_gate_combine(p, self.o_fine_t, self.g_t, self.o_coarse, natural=True, out=self.out,
                         stream=stream)
        return self.out


class LayerPipeline:
    """Layers over host-resident inputs through the library's runner
    (vsa_runner_*): while layer i computes, the inputs of layer i+1 are copied
    in and the output of layer i-1 is copied out (three CUDA streams and two
    buffer sets, all inside the library).  Host tensors must be pinned for
    the copies to run asynchronously.  Each layer's output is bit-identical to
    the fused Layer's."""

    def __init__(self, plan: Plan, B: int, H: int, D: int, k: int, scale: Optional[float] = None,
                 device=None):
        dev = torch.device("cuda", plan.device) if device is None else torch.device(device)
        self.plan, self.dev, self.B, self.H, self.D = plan, dev, B, H, D
        self.scale = D ** -0.5 if scale is None else float(scale)
        h = ctypes.c_void_p()
        with torch.cuda.device(dev):
            _check(lib().vsa_runner_create(plan.handle, B, H, D, k, self.scale, ctypes.byref(h)))
        self._h = h

    def run(self, host_inputs: Sequence[dict], host_outputs: Sequence[torch.Tensor]) -> None:
        """Layer i reads host_inputs[i] (dict of pinned "q", "k", "v", "g"
        [B,H,N,D] bf16) and writes host_outputs[i] (pinned [B,H,N,D] bf16).
        Asynchronous: the current stream waits for the last copy-out."""
        n = len(host_inputs)
        if len(host_outputs) != n:
            raise ValueError("one output per input set")
        shape = (self.B, self.H, self.plan.n_tokens, self.D)
        for t in [*(d[x] for d in host_inputs for x in "qkvg"), *host_outputs]:
            if t.device.type != "cpu" or t.dtype != torch.bfloat16 or tuple(t.shape) != shape \
                    or not t.is_contiguous():
                raise ValueError(f"host tensors must be contiguous CPU bf16 {shape}")
        arr = lambda ts: (ctypes.c_void_p * max(n, 1))(*(t.data_ptr() for t in ts))
        q, k, v, g = (arr([d[x] for d in host_inputs]) for x in "qkvg")
        out = arr(host_outputs)
        with torch.cuda.device(self.dev):
            _check(lib().vsa_runner_run(self._h, n, q, k, v, g, out,
                                        _stream(torch.cuda.current_stream(self.dev))))

    def elapsed_ms(self) -> float:
        """Device time of the last run (first copy-in to last copy-out), in ms."""
        ms = ctypes.c_float()
        _check(lib().vsa_runner_elapsed(self._h, ctypes.byref(ms)))
        return float(ms.value)

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            with torch.cuda.device(self.dev):
                lib().vsa_runner_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class TrainingLayer:
    """Forward and backward of the layer for training.  ``forward`` runs the
    unfused chain and keeps what the backward needs (tiled Q, K, V, G, the
    pooled means, o_coarse, the selection, o_fine and its log-sum-exp);
    ``backward(d_out)`` returns (dq, dk, dv, dg) in natural order [B,H,N,D],
    bf16: permute d_out, combine backward, coarse backward, attention backward
    (with the pooling term), and four unpermutes.  The selection passes no
    gradient.  Buffers are allocated once and reused."""

    def __init__(self, plan: Plan, B: int, H: int, D: int, k: int, scale: Optional[float] = None,
                 device=None, k_ref: Optional[int] = None):
        self.plan, self.B, self.H, self.D, self.k, self.k_ref = plan, B, H, D, k, k_ref
        self.scale = D ** -0.5 if scale is None else float(scale)
        dev = torch.device("cuda", plan.device) if device is None else torch.device(device)
        tiled = (B, H, plan.n_padded, D)
        bf = dict(dtype=torch.bfloat16, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.q_t, self.k_t, self.v_t, self.g_t, self.o_fine_t, self.d_out_t = (
            torch.empty(tiled, **bf) for _ in range(6))
        self.o_coarse = torch.empty(B, H, plan.n_tiles, D, **f32)
        self.lse = torch.empty(B, H, plan.n_padded, **f32)
        self.topk_idx = torch.empty(B, H, plan.n_video_tiles, max(k, 0), dtype=torch.int32, device=dev)
        self.topk_ref = (torch.empty(B, H, plan.n_video_tiles, max(k_ref, 0), dtype=torch.int32, device=dev)
                         if k_ref is not None else None)
        self.ws = torch.empty(max(plan.workspace_size(B, H, D, k), 16), dtype=torch.uint8, device=dev)
        self.bws = torch.empty(max(vsa_backward_workspace_size(plan, B, H, D), 16), dtype=torch.uint8,
                               device=dev)
        self.out = torch.empty(B, H, plan.n_tokens, D, **bf)
        self.delta = torch.empty(B, H, plan.n_padded, **f32)
        self.d_o_coarse = torch.empty(B, H, plan.n_tiles, D, **f32)
        self.d_bar = tuple(torch.empty(B, H, plan.n_tiles, D, **f32) for _ in range(3))
        self.dq_t, self.dk_t, self.dv_t, self.dg_t = (torch.empty(tiled, **bf) for _ in range(4))
        self.grads = tuple(torch.empty(B, H, plan.n_tokens, D, **bf) for _ in range(4))

    def forward(self, q, k, v, g, stream=None):
        p = self.plan
        qbar, kbar, vbar = pooled_slots(p, self.ws, self.B, self.H, self.D)
        vsa_permute_pool(p, q, self.q_t, qbar, stream)
        vsa_permute_pool(p, k, self.k_t, kbar, stream)
        vsa_permute_pool(p, v, self.v_t, vbar, stream)
        vsa_coarse_topk_pooled(p, self.B, self.H, self.D, self.k, self.ws, self.scale,
                               o_coarse=self.o_coarse, topk_idx=self.topk_idx, stream=stream)
        vsa_permute(p, g, self.g_t, stream)
        kr = p.n_prefix_tiles if self.k_ref is None else self.k_ref
        if self.k_ref is not None:
            vsa_select_reference(p, self.B, self.H, self.D, self.k_ref, self.ws, self.scale,
                                 out=self.topk_ref, stream=stream)
        _check(lib().vsa_sparse_attn_ref(
            p.handle, _ptr(self.q_t), _ptr(self.k_t), _ptr(self.v_t),
            _ptr(self.topk_idx) if self.topk_idx.numel() else None, self.k,
            _ptr(self.topk_ref) if self.topk_ref is not None and self.topk_ref.numel() else None, kr,
            self.B, self.H, self.D, self.scale, None, None, _ptr(self.o_fine_t), _ptr(self.lse),
            _stream(stream)))
        vsa_gate_combine(p, self.o_fine_t, self.g_t, self.o_coarse, natural=True, out=self.out,
                         stream=stream)
        return self.out

    def backward(self, d_out, stream=None):
        p = self.plan
        vsa_permute(p, d_out, self.d_out_t, stream)
        vsa_combine_backward(p, self.d_out_t, self.o_fine_t, self.g_t, self.o_coarse, self.delta,
                             self.dg_t, self.d_o_coarse, stream)
        qbar, kbar, vbar = pooled_slots(p, self.ws, self.B, self.H, self.D)
        vsa_coarse_backward(p, qbar, kbar, vbar, self.d_o_coarse, self.bws, self.scale,
                            out=self.d_bar, stream=stream)
        vsa_sparse_attn_backward(p, self.q_t, self.k_t, self.v_t, self.d_out_t, self.topk_idx,
                                 self.k, self.lse, self.delta, self.bws, topk_ref=self.topk_ref,
                                 k_ref=self.k_ref, d_bar=self.d_bar, scale=self.scale,
                                 out=(self.dq_t, self.dk_t, self.dv_t), stream=stream)
        for src, dst in zip((self.dq_t, self.dk_t, self.dv_t, self.dg_t), self.grads):
            vsa_unpermute(p, src, dst, stream)
        return self.grads
