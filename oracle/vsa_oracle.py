"""Plain fp64 CPU oracle for the VSA tile-sparse attention layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product imports this module: only
the tests, the smoke check and the benchmark's CPU-baseline leg call it.  It
shares no code with the CUDA path (no tables, helpers or constants); the two
meet only in the seeded input generator ``tile_sparse_video_b200.inputs``.

Every step is the plain definition, written for a reader to check by eye:
numpy fp64 arithmetic, a matrix product or a sort from the library where the
definition calls for one, and no blocking, fusion or reordering.

Sources ("the pages"):
  [SNACK]  "ComfyUI-Ref2VA-VSA proves a sparse attention gate can be
           transplanted ..." (SnackOnAI analysis): sections "The Architecture,
           Unpacked", "The Code, Annotated" (snippets one, two, four) and
           "It In Action".
  [WIKI]   "Ref2VA VSA: Sparse Attention Node for H3 Reference-to-Video"
           (ComfyUI wiki news): section "The two-tier attention patch".
  [VEDA]   "Veda Sparse Attention" (ComfyUI wiki news, Japanese): the node's
           input table (generated_sparsity) and section "Performance".
  [README] The ComfyUI-Ref2VA-VSA README: "Technical Architecture".

Readings taken where the pages are silent are marked "Reading:" below.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
facts the pages or the mathematics fix (the pages' worked tile counts, an
independent coordinate formula, a library attention routine, closed forms).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


# ---------------------------------------------------------------------------
# Step 1: the geometry plan (segment-pure prefix tiles, then video cubes).
# ---------------------------------------------------------------------------

@dataclass
class Plan:
    R: int                  # rows per tile
    n_tokens: int           # N real tokens (prefix + video)
    n_prefix_tiles: int     # n_p: tiles [0, n_p) hold the prefix
    n_tiles: int            # T
    untile: np.ndarray      # int64[N]: token -> row of the padded tile layout
    row_src: np.ndarray     # int64[T*R]: row -> token, or -1 for a pad row
    block_len: np.ndarray   # int64[T]: live (real) rows of each tile
    tile_seg: np.ndarray    # int64[T]: prefix segment of the tile, -1 = video

    @property
    def n_padded(self) -> int:
        return self.n_tiles * self.R

    @property
    def n_video_tiles(self) -> int:
        return self.n_tiles - self.n_prefix_tiles


def plan(prefix_lens, grid, tile) -> Plan:
    """Build the token -> padded-row map.

    [SNACK] snippet one: every prefix segment (text, reference image, reference
    audio, ...) is cut into tiles of R rows, the last tile of a segment may be
    short, and each segment begins on a fresh tile; the prefix tiles come
    first.  The generated video is flattened t-major, then h, then w, and cut
    into cubes visited in loop order t0, h0, w0 ([WIKI] "3D spatio-temporal
    tiles"; [README] "4x4x4").  Real rows sit at the head of their tile and
    ``block_len`` counts them, so pad rows never enter a score.

    Reading (edge cubes): a grid extent that is not a multiple of the cube
    extent gives clipped, partly filled cubes; this is the only rule that
    reproduces the pages' worked count of 660 video tiles and 43,904 padded
    rows for a 37 x 24 x 42 grid ([SNACK] "It In Action", step two).
    Reading (order inside a cube): lexicographic (t, h, w).  The layer's output
    does not depend on it; it only fixes the permutation table.
    """
    tt, th, tw = (int(v) for v in tile)
    R = tt * th * tw
    Tg, Hg, Wg = (int(v) for v in grid)
    prefix_lens = [int(v) for v in prefix_lens]
    if R <= 0 or min(Tg, Hg, Wg) < 0 or any(v < 0 for v in prefix_lens):
        raise ValueError("bad geometry")
    P = sum(prefix_lens)
    N = P + Tg * Hg * Wg
    untile = np.full(N, -1, dtype=np.int64)
    block_len, tile_seg = [], []

    src = 0
    tile_id = 0
    for seg, length in enumerate(prefix_lens):
        left = length
        while left > 0:
            n = min(R, left)
            untile[src:src + n] = tile_id * R + np.arange(n)
            block_len.append(n)
            tile_seg.append(seg)
            src += n
            left -= n
            tile_id += 1
    n_prefix_tiles = tile_id

    for t0 in range(0, Tg, tt):
        for h0 in range(0, Hg, th):
            for w0 in range(0, Wg, tw):
                ts = np.arange(t0, min(t0 + tt, Tg))
                hs = np.arange(h0, min(h0 + th, Hg))
                ws = np.arange(w0, min(w0 + tw, Wg))
                tok = P + (ts[:, None, None] * Hg + hs[None, :, None]) * Wg + ws[None, None, :]
                tok = tok.reshape(-1)            # lexicographic (t, h, w)
                untile[tok] = tile_id * R + np.arange(tok.size)
                block_len.append(tok.size)
                tile_seg.append(-1)
                tile_id += 1

    T = tile_id
    row_src = np.full(T * R, -1, dtype=np.int64)
    row_src[untile] = np.arange(N)

    # Guard rails as in [SNACK] snippet one: refuse a broken map outright.
    if N and (untile.min() < 0 or np.unique(untile).size != N):
        raise RuntimeError("untile map is not injective")
    if np.count_nonzero(row_src >= 0) != N:
        raise RuntimeError("a token was placed twice or not at all")
    return Plan(R=R, n_tokens=N, n_prefix_tiles=n_prefix_tiles, n_tiles=T,
                untile=untile, row_src=row_src,
                block_len=np.asarray(block_len, dtype=np.int64),
                tile_seg=np.asarray(tile_seg, dtype=np.int64))


def keep_count(n_video_tiles: int, n_prefix_tiles: int, keep_ratio=None,
               keep_tiles=None) -> int:
    """Number k of video key tiles each video query tile keeps.

    Ratio mode: keep_ratio = clamp(1 - sparsity, 0, 1) ([SNACK] snippet two)
    and k = ceil(keep_ratio * n_video).  Reading: ceiling, with a 1e-9 guard
    against binary-fraction artefacts; the pages' own figures (165 and 66 of
    660 tiles at 75 % and 90 %, [SNACK] "It In Action", step three) need it.
    Integer mode ([VEDA] generated_sparsity = 24): keep exactly that many,
    capped at n_video.  Reading: k = 0 is only meaningful when prefix sinks
    exist (else a query tile would have no key at all).
    """
    if keep_tiles is not None and keep_tiles >= 0:
        k = min(int(keep_tiles), n_video_tiles)
    else:
        r = min(1.0, max(0.0, float(keep_ratio)))
        k = min(n_video_tiles, int(math.ceil(r * n_video_tiles - 1e-9)))
    if k == 0 and n_prefix_tiles == 0 and n_video_tiles > 0:
        raise ValueError("no key tile left to attend to")
    return k


def keep_count_ref(n_prefix_tiles: int, keep_ratio=None, keep_tiles=None) -> int:
    """Number of reference (prefix) key tiles each video query tile keeps when
    the reference tiles are thinned too ([VEDA] input table: reference_sparsity
    applies "the same setting" to the reference tokens; 0 % is full attention).
    Reading: the keep rule of ``keep_count`` applied to the n_p reference tiles
    (ratio mode ceil(clamp(keep_ratio, 0, 1) * n_p - 1e-9); integer mode
    min(keep_tiles, n_p)), so keep_ratio = 1 keeps every reference tile."""
    if keep_tiles is not None and keep_tiles >= 0:
        return min(int(keep_tiles), n_prefix_tiles)
    r = min(1.0, max(0.0, float(keep_ratio)))
    return min(n_prefix_tiles, int(math.ceil(r * n_prefix_tiles - 1e-9)))


# ---------------------------------------------------------------------------
# Step 1 (data movement): permute into / out of the padded tile layout.
# ---------------------------------------------------------------------------

def permute(x: np.ndarray, p: Plan) -> np.ndarray:
    """x_t[..., untile[n], :] = x[..., n, :]; pad rows are zero
    ([SNACK] snippet two: ``x_t = zeros(...); x_t[untile] = x``)."""
    out = np.zeros(x.shape[:-2] + (p.n_padded, x.shape[-1]), dtype=x.dtype)
    out[..., p.untile, :] = x
    return out


def unpermute(x_t: np.ndarray, p: Plan) -> np.ndarray:
    """x[..., n, :] = x_t[..., untile[n], :] (pad rows dropped)."""
    return x_t[..., p.untile, :]


# ---------------------------------------------------------------------------
# Step 2: coarse attention over mean-pooled tiles.
# ---------------------------------------------------------------------------

def pool(x_t: np.ndarray, p: Plan) -> np.ndarray:
    """Per-tile mean over the live rows only.

    Reading: the pages name "coarse tile selection" ([SNACK] "References",
    the VSA paper) without defining the pooling; the plainest reading is the
    arithmetic mean of the tile's real tokens (pad rows are excluded,
    [SNACK] snippet two on block_len).
    """
    shp = x_t.shape[:-2]
    out = np.zeros(shp + (p.n_tiles, x_t.shape[-1]), dtype=np.float64)
    for t in range(p.n_tiles):
        rows = x_t[..., t * p.R: t * p.R + p.block_len[t], :].astype(np.float64)
        out[..., t, :] = rows.sum(axis=-2) / p.block_len[t]
    return out


def coarse_attention(qbar, kbar, vbar, scale):
    """Coarse attention of every pooled query tile over every pooled key tile.

    s[i, j] = scale * <qbar_i, kbar_j>;  o_coarse_i = sum_j softmax_j(s_i)_j vbar_j.
    Reading: all T tiles are coarse keys and every query tile (prefix ones
    too) gets a coarse output; softmax is the two-pass max / sum form.
    Returns (s [.., T, T], o_coarse [.., T, D]), fp64.
    """
    s = scale * (qbar @ np.swapaxes(kbar, -1, -2))
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    prob = e / e.sum(axis=-1, keepdims=True)
    return s, prob @ vbar


# ---------------------------------------------------------------------------
# Step 3: per-head top-k over the video key tiles.
# ---------------------------------------------------------------------------

def select_topk(s: np.ndarray, p: Plan, k: int) -> np.ndarray:
    """For each video query tile i (n_p <= i < T) and head: the k video key
    tiles with the highest coarse score s[i, j], ties broken towards the lower
    tile index, returned in ascending tile order ([WIKI] "Sparse video only":
    top-k applies strictly to the generated-video key tiles; [VEDA]
    "head-aware top-k").  Prefix key tiles are never candidates: they are
    always-kept sinks.  Result: int64 [.., n_v, k] of global tile indices.
    """
    n_p, T = p.n_prefix_tiles, p.n_tiles
    lead = s.shape[:-2]
    out = np.zeros(lead + (T - n_p, k), dtype=np.int64)
    cand = np.arange(n_p, T)
    for idx in np.ndindex(*lead):
        for i in range(n_p, T):
            scores = s[idx + (i,)][n_p:]
            # sort by score descending, then by tile index ascending
            order = np.lexsort((cand, -scores))
            out[idx + (i - n_p,)] = np.sort(cand[order[:k]])
    return out


def select_topk_ref(s: np.ndarray, p: Plan, k_ref: int) -> np.ndarray:
    """For each video query tile i and head: the k_ref reference (prefix) key
    tiles with the highest coarse score s[i, j], j < n_p, ties towards the
    lower index, in ascending order.  Reading of [VEDA] reference_sparsity:
    the reference key tiles are thinned by the same per-head top-k as the
    generated-video ones, with their own keep count (``keep_count_ref``);
    reference query tiles stay dense.  Result: int64 [.., n_v, k_ref]."""
    n_p, T = p.n_prefix_tiles, p.n_tiles
    lead = s.shape[:-2]
    out = np.zeros(lead + (T - n_p, k_ref), dtype=np.int64)
    cand = np.arange(n_p)
    for idx in np.ndindex(*lead):
        for i in range(n_p, T):
            order = np.lexsort((cand, -s[idx + (i,)][:n_p]))
            out[idx + (i - n_p,)] = np.sort(cand[order[:k_ref]])
    return out


def key_tiles(p: Plan, i: int, kept_row, kept_ref_row=None) -> np.ndarray:
    """Key tile set of query tile i: all tiles for a prefix query tile (prefix
    queries attend densely, [SNACK] snippet two ``sink_q``); for a video query
    tile the prefix sinks (or, with reference thinning, its kept reference
    tiles ``kept_ref_row``) plus its kept video tiles (``sink_blocks``)."""
    if i < p.n_prefix_tiles:
        return np.arange(p.n_tiles)
    ref = np.arange(p.n_prefix_tiles) if kept_ref_row is None else np.asarray(kept_ref_row, dtype=np.int64)
    return np.concatenate([ref, np.asarray(kept_row, dtype=np.int64)])


# ---------------------------------------------------------------------------
# Step 4: block-sparse fine attention.
# ---------------------------------------------------------------------------

def fine_tile(q_t, k_t, v_t, p: Plan, i: int, tiles, scale):
    """Softmax attention of the live query rows of tile i over the live key
    rows of ``tiles`` (one head: q_t, k_t, v_t are [N_pad, D]).

    Returns (o [block_len[i], D], lse [block_len[i]]) in fp64.
    """
    rows = np.concatenate([j * p.R + np.arange(p.block_len[j]) for j in tiles])
    q = q_t[i * p.R: i * p.R + p.block_len[i]].astype(np.float64)
    kk = k_t[rows].astype(np.float64)
    vv = v_t[rows].astype(np.float64)
    s = scale * (q @ kk.T)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return (e @ vv) / l, (m + np.log(l))[:, 0]


def fine(q_t, k_t, v_t, p: Plan, kept, scale, kept_ref=None):
    """o_fine for every live row of every tile (pad rows zero), and its
    log-sum-exp.  q_t, k_t, v_t: [B, H, N_pad, D]; kept: [B, H, n_v, k];
    kept_ref (optional): [B, H, n_v, k_ref] kept reference tiles."""
    B, H = q_t.shape[:2]
    o = np.zeros(q_t.shape, dtype=np.float64)
    lse = np.zeros(q_t.shape[:-1], dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for i in range(p.n_tiles):
                row = kept[b, h, i - p.n_prefix_tiles] if i >= p.n_prefix_tiles else None
                ref = (kept_ref[b, h, i - p.n_prefix_tiles]
                       if kept_ref is not None and i >= p.n_prefix_tiles else None)
                oi, li = fine_tile(q_t[b, h], k_t[b, h], v_t[b, h], p, i,
                                   key_tiles(p, i, row, ref), scale)
                n = p.block_len[i]
                o[b, h, i * p.R: i * p.R + n] = oi
                lse[b, h, i * p.R: i * p.R + n] = li
    return o, lse


# ---------------------------------------------------------------------------
# Step 5: gated combine.
# ---------------------------------------------------------------------------

def sigmoid(x):
    """Logistic function 1 / (1 + e^-x), in fp64 (e^-x may overflow to inf,
    which gives the correct limit 0)."""
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def gate_combine(o_fine, g_t, o_coarse, p: Plan):
    """out = o_fine + sigmoid(g) * o_coarse[tile(row)] on live rows, 0 on pads.

    g is the bias-free ``to_gate_compress`` projection of the layer input,
    split into heads ([SNACK] snippet two: ``gate_t`` viewed as
    [1, S_pad, heads, head_dim] and passed as ``coarse_gate``).  Reading: the
    gate weighs the coarse branch element-wise through a logistic sigmoid.
    """
    tile_of_row = np.repeat(np.arange(p.n_tiles), p.R)
    live = p.row_src >= 0
    out = o_fine + sigmoid(g_t.astype(np.float64)) * o_coarse[..., tile_of_row, :]
    out[..., ~live, :] = 0.0
    return out


def project(x, w, n_heads: int, head_dim: int, act=None):
    """Bias-free linear of the layer input, split into heads:
    y[b, h, n, d] = act( sum_c x[b, n, c] * w[h*head_dim + d, c] ).

    The gate is such a projection: [SNACK] snippet two computes ``gate_t`` as
    ``to_gate_compress(x_t)`` viewed as [1, S, heads, head_dim], and snippet
    three installs ``to_gate_compress`` as an ``nn.Linear`` without bias (weight
    layout [out = heads*head_dim, in = width]).  ``act`` is None or "sigmoid".
    x: [B, N, C], w: [H*D, C], any float dtype (converted exactly to fp64);
    returns fp64 [B, H, N, D].
    """
    xf, wf = as_f64(x), as_f64(w)
    y = xf @ wf.T                                        # [B, N, H*D]
    B, N = y.shape[0], y.shape[1]
    y = y.reshape(B, N, n_heads, head_dim).transpose(0, 2, 1, 3)
    return sigmoid(y) if act == "sigmoid" else y


# ---------------------------------------------------------------------------
# The whole layer.
# ---------------------------------------------------------------------------

def as_f64(x) -> np.ndarray:
    """Exact conversion of an input (numpy array or torch tensor, e.g. bf16)
    to a float64 numpy array."""
    if type(x).__module__.split(".")[0] == "torch":
        import torch
        return x.detach().to(device="cpu", dtype=torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def layer(q, k, v, g, p: Plan, kk: int, scale=None, kept=None, k_ref=None, kept_ref=None):
    """Steps 1-5 on natural-order inputs [B, H, N, D] (any float dtype,
    converted exactly to fp64).  ``kept`` overrides the top-k selection (used
    to evaluate the oracle under another legal tie-break).  ``k_ref`` (None:
    every reference tile is a sink) thins the reference key tiles of video
    query tiles to their top k_ref; ``kept_ref`` overrides that selection.
    Returns a dict of every intermediate, all fp64 except the integer
    selections."""
    D = q.shape[-1]
    scale = D ** -0.5 if scale is None else scale
    q_t, k_t, v_t, g_t = (permute(as_f64(x), p) for x in (q, k, v, g))
    qbar, kbar, vbar = pool(q_t, p), pool(k_t, p), pool(v_t, p)
    s, o_coarse = coarse_attention(qbar, kbar, vbar, scale)
    sel = select_topk(s, p, kk) if kept is None else np.asarray(kept, dtype=np.int64)
    sel_ref = None
    if kept_ref is not None:
        sel_ref = np.asarray(kept_ref, dtype=np.int64)
    elif k_ref is not None:
        sel_ref = select_topk_ref(s, p, k_ref)
    o_fine, lse = fine(q_t, k_t, v_t, p, sel, scale, sel_ref)
    out_t = gate_combine(o_fine, g_t, o_coarse, p)
    return dict(q_t=q_t, k_t=k_t, v_t=v_t, g_t=g_t, qbar=qbar, kbar=kbar, vbar=vbar,
                scores=s, o_coarse=o_coarse, topk=sel, topk_ref=sel_ref, o_fine=o_fine, lse=lse,
                out_t=out_t, out=unpermute(out_t, p))


# ---------------------------------------------------------------------------
# The backward pass: gradients of a scalar loss through steps 5 .. 1.
#
# The method is trained end to end ([SNACK] "The Architecture, Unpacked":
# the coarse stage and the gate are learned; the VSA paper it builds on
# trains the sparse kernel).  Reading: the top-k selection is an index choice
# and passes no gradient (it is piecewise constant in the scores); gradients
# flow through the coarse branch (pooling, coarse attention), the fine
# attention over the selected tiles and the gate.  Every function takes the
# upstream gradient of its output and returns the gradients of its inputs,
# written from the definitions of the forward steps above.
# ---------------------------------------------------------------------------

def gate_combine_backward(d_out_t, o_fine, g_t, o_coarse, p: Plan):
    """Backward of out = o_fine + sigmoid(g) * o_coarse[tile(row)] (live rows).

    Returns (d_o_fine [.., N_pad, D], d_g_t [.., N_pad, D],
    d_o_coarse [.., T, D]); pad rows carry no gradient.
    """
    tile_of_row = np.repeat(np.arange(p.n_tiles), p.R)
    live = p.row_src >= 0
    d = np.array(d_out_t, dtype=np.float64)
    d[..., ~live, :] = 0.0
    sg = sigmoid(g_t.astype(np.float64))
    d_o_fine = d.copy()
    d_g_t = d * o_coarse[..., tile_of_row, :] * sg * (1.0 - sg)
    d_o_coarse = np.zeros(o_coarse.shape, dtype=np.float64)
    for t in range(p.n_tiles):
        rows = slice(t * p.R, t * p.R + p.block_len[t])
        d_o_coarse[..., t, :] = (d[..., rows, :] * sg[..., rows, :]).sum(axis=-2)
    return d_o_fine, d_g_t, d_o_coarse


def softmax_backward(prob, d_prob):
    """Row-wise softmax Jacobian applied to an upstream gradient:
    d_s = prob * (d_prob - sum_j prob_j d_prob_j)."""
    return prob * (d_prob - (prob * d_prob).sum(axis=-1, keepdims=True))


def fine_tile_backward(q_t, k_t, v_t, p: Plan, i: int, tiles, scale, d_o):
    """Backward of ``fine_tile`` for one head: given d_o [block_len[i], D],
    the gradients of the query rows of tile i and of the key / value rows
    of ``tiles`` (as (rows, dq, dk, dv): the key rows in ``tiles`` order)."""
    rows = np.concatenate([j * p.R + np.arange(p.block_len[j]) for j in tiles])
    q = q_t[i * p.R: i * p.R + p.block_len[i]].astype(np.float64)
    kk = k_t[rows].astype(np.float64)
    vv = v_t[rows].astype(np.float64)
    s = scale * (q @ kk.T)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    prob = e / e.sum(axis=1, keepdims=True)
    dv = prob.T @ d_o
    d_s = softmax_backward(prob, d_o @ vv.T)
    dq = scale * (d_s @ kk)
    dk = scale * (d_s.T @ q)
    return rows, dq, dk, dv


def fine_backward(q_t, k_t, v_t, p: Plan, kept, scale, d_o_fine, kept_ref=None):
    """Backward of ``fine``: gradients of q_t, k_t, v_t [B, H, N_pad, D]
    (pad rows zero) for the upstream d_o_fine, under the fixed selection."""
    B, H = q_t.shape[:2]
    dq = np.zeros(q_t.shape, dtype=np.float64)
    dk = np.zeros(k_t.shape, dtype=np.float64)
    dv = np.zeros(v_t.shape, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for i in range(p.n_tiles):
                row = kept[b, h, i - p.n_prefix_tiles] if i >= p.n_prefix_tiles else None
                ref = (kept_ref[b, h, i - p.n_prefix_tiles]
                       if kept_ref is not None and i >= p.n_prefix_tiles else None)
                qrows = slice(i * p.R, i * p.R + p.block_len[i])
                rows, dqi, dki, dvi = fine_tile_backward(
                    q_t[b, h], k_t[b, h], v_t[b, h], p, i, key_tiles(p, i, row, ref), scale,
                    np.asarray(d_o_fine[b, h, qrows], dtype=np.float64))
                dq[b, h, qrows] += dqi
                np.add.at(dk[b, h], rows, dki)
                np.add.at(dv[b, h], rows, dvi)
    return dq, dk, dv


def coarse_attention_backward(qbar, kbar, vbar, scale, d_o_coarse):
    """Backward of ``coarse_attention``: (d_qbar, d_kbar, d_vbar), fp64."""
    s = scale * (qbar @ np.swapaxes(kbar, -1, -2))
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    prob = e / e.sum(axis=-1, keepdims=True)
    d_vbar = np.swapaxes(prob, -1, -2) @ d_o_coarse
    d_s = softmax_backward(prob, d_o_coarse @ np.swapaxes(vbar, -1, -2))
    d_qbar = scale * (d_s @ kbar)
    d_kbar = scale * (np.swapaxes(d_s, -1, -2) @ qbar)
    return d_qbar, d_kbar, d_vbar


def pool_backward(d_bar, p: Plan):
    """Backward of ``pool``: each live row of tile t receives d_bar[t] /
    block_len[t]; pad rows receive nothing.  Returns [.., N_pad, D]."""
    out = np.zeros(d_bar.shape[:-2] + (p.n_padded, d_bar.shape[-1]), dtype=np.float64)
    for t in range(p.n_tiles):
        n = p.block_len[t]
        out[..., t * p.R: t * p.R + n, :] = d_bar[..., t: t + 1, :] / n
    return out


def layer_backward(d_out, fwd: dict, p: Plan, scale=None):
    """Gradients of the loss sum(d_out * out) with respect to the natural-order
    inputs q, k, v, g [B, H, N, D] of ``layer`` (``fwd`` is its result), under
    the forward's selection.  Returns a dict with dq, dk, dv, dg (natural
    order) and the tiled intermediates, all fp64."""
    D = fwd["q_t"].shape[-1]
    scale = D ** -0.5 if scale is None else scale
    d_out_t = permute(as_f64(d_out), p)
    d_o_fine, d_g_t, d_o_coarse = gate_combine_backward(d_out_t, fwd["o_fine"], fwd["g_t"],
                                                        fwd["o_coarse"], p)
    dq_f, dk_f, dv_f = fine_backward(fwd["q_t"], fwd["k_t"], fwd["v_t"], p, fwd["topk"], scale,
                                     d_o_fine, fwd["topk_ref"])
    d_qbar, d_kbar, d_vbar = coarse_attention_backward(fwd["qbar"], fwd["kbar"], fwd["vbar"],
                                                       scale, d_o_coarse)
    dq_t = dq_f + pool_backward(d_qbar, p)
    dk_t = dk_f + pool_backward(d_kbar, p)
    dv_t = dv_f + pool_backward(d_vbar, p)
    return dict(d_out_t=d_out_t, d_o_fine=d_o_fine, d_o_coarse=d_o_coarse,
                d_qbar=d_qbar, d_kbar=d_kbar, d_vbar=d_vbar,
                dq_t=dq_t, dk_t=dk_t, dv_t=dv_t, dg_t=d_g_t,
                dq=unpermute(dq_t, p), dk=unpermute(dk_t, p), dv=unpermute(dv_t, p),
                dg=unpermute(d_g_t, p))
