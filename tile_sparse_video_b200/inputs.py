"""Seeded synthetic workloads for the VSA tile-sparse attention layer.

This module only draws numbers: it holds none of the layer's arithmetic (no
tiling, pooling, scoring, selection, attention or gating).  Both the fp64
oracle and the CUDA path take their inputs from here, so the two see the very
same bf16 bytes.

Shapes follow the pages' workloads (MiniMax H3 reference-to-video with a
segmented prefix, and the Veda long clip with 128-token key tiles; see
"ComfyUI-Ref2VA-VSA proves a sparse attention gate can be transplanted",
section "It In Action", and the Veda news page, section "Performance").

Recipe (per batch element b, CPU ``torch.Generator`` seeded with
``seed_base + 17*b``; fp32 ``randn`` then round-to-nearest-even to bf16):

* ``values="iid"``: Q, K, V ~ N(0, 1), drawn head by head in that order.
* ``values="head_scaled"``: first a per-head scale s_h ~ U[0.5, 2]; then
  Q, K, V ~ s_h * N(0, 1), head by head.
* ``values="low_rank"``: first a per-head field F ~ N(0, 1) of shape
  [ceil(T/tt), ceil(H/th), ceil(W/tw), 16] over the video tile grid; then for
  Q and for K (each with its own A ~ N(0, 1/16) of shape [16, D] and its own
  noise eps ~ N(0, 1)): prefix rows ~ N(0, 1), video rows
  (F[cell(t,h,w)] @ A + 0.5*eps) / sqrt(1.25); V ~ N(0, 1).  The field makes
  the coarse scores non-uniform, like a real clip.
* gate ``"projected"``: x ~ N(0, 1) of shape [N, C] and W ~ N(0, std^2) of
  shape [H*D, C] (a bias-free linear, out = H*D, in = C); G = x @ W^T
  evaluated in fp64 then rounded to bf16, split into heads.
* gate ``"marginal"``: G ~ N(0, std^2 * C) directly, which is the exact
  marginal law of x @ W^T for the two laws above (saves a host GEMM).

Tensors are returned in natural token order, shape [B, H, N, D], bf16,
contiguous, on the CPU, under keys "q", "k", "v", "g"; "value_scale" [B, H]
holds s_h (1.0 without per-head scaling).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import torch


@dataclass(frozen=True)
class Workload:
    """One synthetic layer invocation: shapes, keep rule and value recipe."""

    name: str
    B: int
    H: int
    D: int
    prefix: tuple            # prefix segment lengths, in sequence order
    grid: tuple              # video latent grid (T, H, W), flattened t-major
    tile: tuple              # video tile shape (tt, th, tw); R = tt*th*tw rows
    sparsity: Optional[float] = None   # ratio mode: keep ceil((1-s) * n_video)
    keep_tiles: Optional[int] = None   # integer mode: keep exactly this many
    values: str = "iid"
    gate: str = "marginal"
    gate_width: int = 64
    gate_std: float = 0.01
    seed_base: int = 0

    @property
    def tile_rows(self) -> int:
        return self.tile[0] * self.tile[1] * self.tile[2]

    @property
    def n_prefix(self) -> int:
        return int(sum(self.prefix))

    @property
    def n_video(self) -> int:
        return self.grid[0] * self.grid[1] * self.grid[2]

    @property
    def n_tokens(self) -> int:
        return self.n_prefix + self.n_video

    @property
    def keep_ratio(self) -> Optional[float]:
        if self.sparsity is None:
            return None
        return min(1.0, max(0.0, 1.0 - self.sparsity))


# The four named workloads.  Sizes are those of the pages' runs: a tiny case
# the oracle finishes instantly, a small H3-like case, a reference-to-video
# layer at H3 width (42 heads x 128 = 5376), and the 104k-token Veda layer.
TINY = Workload("tiny_h2_d64", B=1, H=2, D=64, prefix=(40, 70), grid=(4, 8, 8),
                tile=(4, 4, 4), keep_tiles=2, values="iid", gate="projected",
                gate_width=64, gate_std=0.02, seed_base=1000)
SMALL = Workload("small_h8_9772tok", B=1, H=8, D=128, prefix=(256, 1024, 300),
                 grid=(8, 32, 32), tile=(4, 4, 4), sparsity=0.75, values="iid",
                 gate="projected", gate_width=1024, gate_std=0.01, seed_base=2000)
REF2VA = Workload("ref2va_h42_33920tok", B=1, H=42, D=128,
                  prefix=(512, 256, 256, 256, 256, 128), grid=(32, 24, 42),
                  tile=(4, 4, 4), sparsity=0.75, values="head_scaled",
                  gate="marginal", gate_width=5376, gate_std=0.01, seed_base=3000)
VEDA_104K = Workload("veda_h42_104704tok", B=1, H=42, D=128, prefix=(256,),
                     grid=(32, 48, 68), tile=(4, 8, 4), sparsity=0.90,
                     values="low_rank", gate="marginal", gate_width=5376,
                     gate_std=0.01, seed_base=4000)

WORKLOADS = {w.name: w for w in (TINY, SMALL, REF2VA, VEDA_104K)}


def sweep_workloads() -> list:
    """Sparsity and length sweep over the small and reference-to-video shapes.

    Sparsity 0.50 / 0.75 / 0.90 / 0.95 and an integer keep count of 24, at
    video lengths T x 32 x 32 (T in 16, 32, 64, 102) and T x 24 x 42
    (T in 16, 32, 64, 104); B = 2 (a classifier-free-guidance pair with its
    own seed per element).
    """
    out = []
    seed = 5000
    for base, temporal in ((SMALL, (16, 32, 64, 102)), (REF2VA, (16, 32, 64, 104))):
        for t in temporal:
            grid = (t, base.grid[1], base.grid[2])
            for sp in (0.50, 0.75, 0.90, 0.95, None):
                keep = 24 if sp is None else None
                tag = f"k24" if sp is None else f"s{int(round(sp * 100)):02d}"
                out.append(replace(base, name=f"{base.name.split('_')[0]}_T{t}_{tag}_b2",
                                   B=2, grid=grid, sparsity=sp, keep_tiles=keep,
                                   seed_base=seed))
                seed += 100
    return out


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def _video_cells(w: Workload) -> torch.Tensor:
    """Index of the field cell (t//tt, h//th, w//tw) of every video token, in
    natural (t-major, then h, then w) order."""
    T, Hg, Wg = w.grid
    tt, th, tw = w.tile
    nh, nw = -(-Hg // th), -(-Wg // tw)
    t = torch.arange(T).view(T, 1, 1) // tt
    h = torch.arange(Hg).view(1, Hg, 1) // th
    x = torch.arange(Wg).view(1, 1, Wg) // tw
    return ((t * nh + h) * nw + x).reshape(-1)


def make_inputs(w: Workload, batch: Optional[Sequence[int]] = None,
                heads: Optional[Sequence[int]] = None) -> dict:
    """Draw Q, K, V, G for workload ``w`` (bf16, natural order, [B,H,N,D]).

    ``batch`` / ``heads`` restrict the output to a subset (the draws of the
    skipped heads still happen, so a subset is bit-identical to the same slice
    of the full tensors).
    """
    bsel = list(range(w.B)) if batch is None else list(batch)
    hsel = list(range(w.H)) if heads is None else list(heads)
    N, D, P = w.n_tokens, w.D, w.n_prefix
    shape = (len(bsel), len(hsel), N, D)
    out = {k: torch.empty(shape, dtype=torch.bfloat16) for k in ("q", "k", "v", "g")}
    # per-(b, h) value scale (1 unless values == "head_scaled"); returned so a
    # comparison can state its tolerance per unit of value scale
    out["value_scale"] = torch.ones(len(bsel), len(hsel), dtype=torch.float64)
    cells = _video_cells(w) if w.values == "low_rank" else None
    tt, th, tw = w.tile
    n_cells = (-(-w.grid[0] // tt)) * (-(-w.grid[1] // th)) * (-(-w.grid[2] // tw))
    for bi, b in enumerate(bsel):
        gen = torch.Generator().manual_seed(w.seed_base + 17 * b)
        scale = None
        field_ = None
        if w.values == "head_scaled":
            scale = 0.5 + 1.5 * torch.rand(w.H, generator=gen)
            out["value_scale"][bi] = scale[hsel].double()
        if w.values == "low_rank":
            field_ = torch.randn(w.H, n_cells, 16, generator=gen)
        for name in ("q", "k", "v"):
            for h in range(w.H):
                if w.values == "low_rank" and name != "v":
                    a = torch.randn(16, D, generator=gen) / 4.0
                    pre = torch.randn(P, D, generator=gen)
                    eps = torch.randn(w.n_video, D, generator=gen)
                    vid = (field_[h][cells] @ a + 0.5 * eps) / math.sqrt(1.25)
                    x = torch.cat([pre, vid], 0)
                else:
                    x = torch.randn(N, D, generator=gen)
                    if scale is not None:
                        x = x * scale[h]
                if h in hsel:
                    out[name][bi, hsel.index(h)] = _bf16(x)
        if w.gate == "projected":
            x = torch.randn(N, w.gate_width, generator=gen)
            wt = torch.randn(w.H * D, w.gate_width, generator=gen) * w.gate_std
            g = (x.double() @ wt.double().T).view(N, w.H, D).permute(1, 0, 2)
            for hi, h in enumerate(hsel):
                out["g"][bi, hi] = _bf16(g[h])
        else:
            sigma = w.gate_std * math.sqrt(w.gate_width)
            for h in range(w.H):
                x = torch.randn(N, D, generator=gen) * sigma
                if h in hsel:
                    out["g"][bi, hsel.index(h)] = _bf16(x)
    return out


def make_projection_inputs(w: Workload, batch: Optional[Sequence[int]] = None) -> dict:
    """Draw the inputs of a head projection for workload ``w``: the layer input
    x ~ N(0, 1) [B, N, C] and a bias-free weight W ~ N(0, gate_std^2)
    [H*D, C], C = gate_width, both rounded to bf16 (the gate projection's
    shapes; its own seed stream, separate from Q/K/V/G)."""
    bsel = list(range(w.B)) if batch is None else list(batch)
    N, C, HD = w.n_tokens, w.gate_width, w.H * w.D
    gen = torch.Generator().manual_seed(w.seed_base + 7777)
    weight = _bf16(torch.randn(HD, C, generator=gen) * w.gate_std)
    x = torch.empty(len(bsel), N, C, dtype=torch.bfloat16)
    for bi, b in enumerate(bsel):
        g = torch.Generator().manual_seed(w.seed_base + 7777 + 17 * (b + 1))
        x[bi] = _bf16(torch.randn(N, C, generator=g))
    return {"x": x, "w": weight}


def make_grad_output(w: Workload, batch: Optional[Sequence[int]] = None,
                     heads: Optional[Sequence[int]] = None) -> torch.Tensor:
    """Upstream gradient d_out of the layer output for the backward pass:
    bf16 [B,H,N,D] natural order, N(0, 1), from its own generator per batch
    element (seed ``seed_base + 17*b + 5``), drawn head by head."""
    bsel = list(range(w.B)) if batch is None else list(batch)
    hsel = list(range(w.H)) if heads is None else list(heads)
    out = torch.empty(len(bsel), len(hsel), w.n_tokens, w.D, dtype=torch.bfloat16)
    for bi, b in enumerate(bsel):
        gen = torch.Generator().manual_seed(w.seed_base + 17 * b + 5)
        for h in range(w.H):
            x = torch.randn(w.n_tokens, w.D, generator=gen)
            if h in hsel:
                out[bi, hsel.index(h)] = _bf16(x)
    return out
