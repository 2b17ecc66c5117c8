"""Pins for the fp64 oracle: facts fixed by the pages or by the mathematics,
computed without the oracle's own code paths.

* the pages' worked example (tile counts, padded rows, kept-pair fractions);
* an independent closed-form coordinate formula for token -> padded row;
* a library attention routine (torch scaled_dot_product_attention, fp64) for
  the coarse stage and, at k = all tiles, for the whole fine stage;
* brute-force rank counting for top-k with planted ties;
* closed forms of the softmax and of the gate.
The last block plants mistakes in the oracle and checks that a pin catches
each one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sdpa64(q, k, v, scale):
    """Library softmax attention in fp64 (rows of q over rows of k, v)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    out = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale)
    return out.numpy()


def coord_rows(prefix, grid, tile):
    """Independent closed form of the padded row of every token.

    Prefix token j of segment s: tile = (tiles of earlier segments) + j // R,
    slot j % R.  Video token (t, h, w): cube (t//tt, h//th, w//tw) in t-major
    cube order after the prefix tiles; slot = lexicographic rank inside the
    (clipped) cube.  Returns (row per token, tile per token, tiles per
    prefix, video tile count)."""
    tt, th, tw = tile
    R = tt * th * tw
    rows, tiles = [], []
    base = 0
    for L in prefix:
        for j in range(L):
            rows.append((base + j // R) * R + j % R)
            tiles.append(base + j // R)
        base += -(-L // R)
    n_p = base
    Tg, Hg, Wg = grid
    nH, nW = -(-Hg // th), -(-Wg // tw)
    for t in range(Tg):
        for h in range(Hg):
            for w in range(Wg):
                cube = ((t // tt) * nH + h // th) * nW + w // tw
                bh = min(th, Hg - (h // th) * th)
                bw = min(tw, Wg - (w // tw) * tw)
                slot = ((t % tt) * bh + (h % th)) * bw + (w % tw)
                rows.append((n_p + cube) * R + slot)
                tiles.append(n_p + cube)
    n_v = (-(-Tg // tt)) * nH * nW
    return np.array(rows), np.array(tiles), n_p, n_v


GEOMETRIES = [
    ((40, 70), (4, 8, 8), (4, 4, 4)),
    ((5, 0, 64, 65), (5, 6, 7), (4, 4, 4)),      # empty segment, ragged cubes
    ((), (4, 4, 4), (4, 4, 4)),                   # no prefix
    ((130,), (0, 4, 4), (4, 4, 4)),               # no video
    ((256, 3), (8, 17, 9), (4, 8, 4)),            # 128-row tiles, ragged h and w
    ((1, 1, 1), (3, 3, 3), (4, 4, 4)),            # every tile partial
]


# --------------------------------------------------------------------------
# Plan
# --------------------------------------------------------------------------

def test_plan_reproduces_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "h3_worked_example.json")))
    # the pages' token arithmetic for 1344x768, 124 frames
    F, W, H = g["frames"], g["width"], g["height"]
    lt = ((F - 5) // 17) * 5 + 2
    assert [lt, H // 16 // 2, W // 16 // 2] == g["grid"]
    assert [150, 24 * 42, round(F / 24 * 40) * 2] == g["prefix_lens"]
    p = O.plan(g["prefix_lens"], g["grid"], g["tile"])
    assert p.n_tokens == g["n_tokens"]
    assert p.n_tokens - sum(g["prefix_lens"]) == g["n_video_tokens"]
    assert p.n_prefix_tiles == g["n_prefix_tiles"]
    assert p.n_video_tiles == g["n_video_tiles"]
    assert p.n_padded == g["n_padded_rows"]


@pytest.mark.parametrize("prefix,grid,tile", GEOMETRIES)
def test_plan_matches_coordinate_formula(prefix, grid, tile):
    p = O.plan(prefix, grid, tile)
    rows, tiles, n_p, n_v = coord_rows(prefix, grid, tile)
    assert p.n_prefix_tiles == n_p
    assert p.n_tiles == n_p + n_v
    assert np.array_equal(p.untile, rows)
    # block_len = number of tokens that fall in each tile
    assert np.array_equal(p.block_len, np.bincount(tiles, minlength=p.n_tiles))


@pytest.mark.parametrize("prefix,grid,tile", GEOMETRIES)
def test_plan_invariants(prefix, grid, tile):
    p = O.plan(prefix, grid, tile)
    N = p.n_tokens
    assert np.unique(p.untile).size == N                      # injective
    assert np.array_equal(p.row_src[p.untile], np.arange(N))  # inverse
    seg_of_token = np.concatenate([np.full(L, s) for s, L in enumerate(prefix)] +
                                  [np.full(N - sum(prefix), -1)]).astype(np.int64)
    for t in range(p.n_tiles):
        src = p.row_src[t * p.R:(t + 1) * p.R]
        live = src[src >= 0]
        assert p.block_len[t] >= 1
        assert live.size == p.block_len[t]
        assert np.all(src[:live.size] >= 0) and np.all(src[live.size:] < 0)  # pads at the tail
        assert np.all(seg_of_token[live] == p.tile_seg[t])                 # segment purity
    assert np.all(p.tile_seg[:p.n_prefix_tiles] >= 0)
    assert np.all(p.tile_seg[p.n_prefix_tiles:] == -1)


def test_keep_count_and_pair_fractions_match_pages():
    g = json.load(open(os.path.join(GOLDEN, "h3_worked_example.json")))
    n_p, n_v = g["n_prefix_tiles"], g["n_video_tiles"]
    T = n_p + n_v
    for case in g["keep"]:
        k = O.keep_count(n_v, n_p, keep_ratio=1.0 - case["sparsity"])
        if "k" in case:
            assert k == case["k"]
        pairs = n_v * (n_p + k) + n_p * T      # video rows: sinks + kept; prefix rows: dense
        assert round(pairs / T ** 2, 3) == case["pair_fraction"]


def test_keep_count_modes():
    assert O.keep_count(816, 2, keep_ratio=0.10) == 82
    assert O.keep_count(20, 1, keep_ratio=1 - 0.95) == 1       # (1-0.95)*20 is 0.99999...
    assert O.keep_count(660, 26, keep_tiles=24) == 24
    assert O.keep_count(10, 26, keep_tiles=24) == 10
    assert O.keep_count(10, 1, keep_ratio=0.0) == 0
    assert O.keep_count(10, 1, keep_ratio=2.0) == 10
    with pytest.raises(ValueError):
        O.keep_count(10, 0, keep_ratio=0.0)


def test_permute_roundtrip_and_zero_pads():
    p = O.plan((5, 0, 64, 65), (5, 6, 7), (4, 4, 4))
    x = np.random.default_rng(0).standard_normal((2, 3, p.n_tokens, 8))
    xt = O.permute(x, p)
    assert np.array_equal(O.unpermute(xt, p), x)
    assert np.all(xt[..., p.row_src < 0, :] == 0)


# --------------------------------------------------------------------------
# Pool and coarse attention
# --------------------------------------------------------------------------

def test_pool_is_mean_of_tile_tokens():
    prefix, grid, tile = (5, 0, 64, 65), (5, 6, 7), (4, 4, 4)
    p = O.plan(prefix, grid, tile)
    _, tiles, _, _ = coord_rows(prefix, grid, tile)
    x = np.random.default_rng(1).standard_normal((2, p.n_tokens, 8))
    pooled = O.pool(O.permute(x, p), p)
    for t in range(p.n_tiles):
        np.testing.assert_allclose(pooled[:, t], x[:, tiles == t].mean(axis=1), rtol=1e-13, atol=1e-14)


def test_coarse_matches_library_attention():
    rng = np.random.default_rng(2)
    q, k, v = (rng.standard_normal((2, 3, 11, 16)) for _ in range(3))
    s, oc = O.coarse_attention(q, k, v, 0.25)
    np.testing.assert_allclose(oc, sdpa64(q, k, v, 0.25), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s[1, 2, 4, 7], 0.25 * sum(q[1, 2, 4, d] * k[1, 2, 7, d] for d in range(16)),
                               rtol=1e-12)


def test_coarse_closed_forms():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((1, 1, 1, 4))
    _, oc = O.coarse_attention(rng.standard_normal((1, 1, 1, 4)), rng.standard_normal((1, 1, 1, 4)), v, 1.0)
    np.testing.assert_allclose(oc, v, rtol=1e-15)                 # one key tile: o = v
    v = rng.standard_normal((1, 1, 6, 4))
    _, oc = O.coarse_attention(np.zeros((1, 1, 5, 4)), rng.standard_normal((1, 1, 6, 4)), v, 1.0)
    np.testing.assert_allclose(oc, np.broadcast_to(v.mean(axis=2, keepdims=True), oc.shape), rtol=1e-13)


# --------------------------------------------------------------------------
# Top-k
# --------------------------------------------------------------------------

def brute_topk(scores, k):
    """Rank counting: j is kept iff fewer than k candidates beat it, where j'
    beats j when its score is higher, or equal with a lower index."""
    n = scores.size
    keep = [j for j in range(n)
            if sum(1 for jj in range(n) if scores[jj] > scores[j] or
                   (scores[jj] == scores[j] and jj < j)) < k]
    return np.array(keep)


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    p = O.plan((10, 70), (8, 8, 12), (4, 4, 4))          # n_v = 12
    T, n_p = p.n_tiles, p.n_prefix_tiles
    s = rng.integers(0, 4, size=(2, T, T)).astype(np.float64)   # many exact ties
    for k in (0, 1, 3, 7, p.n_video_tiles):
        sel = O.select_topk(s, p, k)
        for h in range(2):
            for i in range(n_p, T):
                want = n_p + brute_topk(s[h, i, n_p:], k)
                assert np.array_equal(sel[h, i - n_p], want)


@pytest.mark.parametrize("seed", [0, 1])
def test_reference_topk_matches_brute_force_with_ties(seed):
    rng = np.random.default_rng(100 + seed)
    p = O.plan((64, 64, 64, 64, 30), (4, 8, 8), (4, 4, 4))   # n_p = 5 reference tiles
    T, n_p = p.n_tiles, p.n_prefix_tiles
    s = rng.integers(0, 3, size=(2, T, T)).astype(np.float64)   # many exact ties
    for k_ref in (0, 1, 2, 4, n_p):
        sel = O.select_topk_ref(s, p, k_ref)
        for h in range(2):
            for i in range(n_p, T):
                assert np.array_equal(sel[h, i - n_p], brute_topk(s[h, i, :n_p], k_ref))


def test_reference_keep_count():
    # 26 reference tiles (the pages' H3 prefix) at 90 % -> 3; at 0 % -> all (full attention)
    assert O.keep_count_ref(26, keep_ratio=0.10) == 3
    assert O.keep_count_ref(26, keep_ratio=1.0) == 26
    assert O.keep_count_ref(2, keep_ratio=0.10) == 1
    assert O.keep_count_ref(26, keep_tiles=24) == 24 and O.keep_count_ref(5, keep_tiles=24) == 5


def test_reference_thinning_reduces_and_restricts():
    """k_ref = n_p keeps every reference tile: the layer is the unthinned one.
    With k_ref < n_p a video query row attends exactly to the tokens of its
    kept reference tiles and kept video tiles (library attention over them)."""
    prefix, grid, tile = (40, 70, 30), (8, 8, 8), (4, 4, 4)
    p = O.plan(prefix, grid, tile)
    _, tiles, _, _ = coord_rows(prefix, grid, tile)
    rng = np.random.default_rng(9)
    q, k, v, g = (rng.standard_normal((1, 2, p.n_tokens, 16)) for _ in range(4))
    base = O.layer(q, k, v, g, p, 3, scale=0.25)
    full = O.layer(q, k, v, g, p, 3, scale=0.25, k_ref=p.n_prefix_tiles)
    np.testing.assert_array_equal(full["out"], base["out"])
    res = O.layer(q, k, v, g, p, 3, scale=0.25, k_ref=1)
    of = O.unpermute(res["o_fine"], p)
    n_prefix_tok = sum(prefix)
    np.testing.assert_array_equal(of[:, :, :n_prefix_tok], O.unpermute(base["o_fine"], p)[:, :, :n_prefix_tok])
    for h in range(2):
        for n in range(n_prefix_tok, p.n_tokens, 11):
            i = tiles[n]
            allowed = (set(res["topk_ref"][0, h, i - p.n_prefix_tiles].tolist())
                       | set(res["topk"][0, h, i - p.n_prefix_tiles].tolist()))
            keys = np.array([m for m in range(p.n_tokens) if tiles[m] in allowed])
            want = sdpa64(q[0, h, n:n + 1], k[0, h, keys], v[0, h, keys], 0.25)
            np.testing.assert_allclose(of[0, h, n:n + 1], want, rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# Fine attention
# --------------------------------------------------------------------------

def _natural_dense(q, k, v, scale):
    """Dense attention of every real token over every real token, natural
    order, by the library routine."""
    return sdpa64(q, k, v, scale)


@pytest.mark.parametrize("prefix,grid,tile", [((40, 70), (4, 8, 8), (4, 4, 4)),
                                               ((5, 0, 64, 65), (5, 6, 7), (4, 4, 4)),
                                               ((3,), (4, 9, 5), (4, 8, 4))])
def test_fine_at_full_keep_is_dense_attention(prefix, grid, tile):
    p = O.plan(prefix, grid, tile)
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((1, 2, p.n_tokens, 16)) for _ in range(3))
    g = rng.standard_normal((1, 2, p.n_tokens, 16))
    res = O.layer(q, k, v, g, p, p.n_video_tiles, scale=0.3)
    np.testing.assert_allclose(O.unpermute(res["o_fine"], p), _natural_dense(q, k, v, 0.3),
                               rtol=1e-11, atol=1e-12)
    assert np.all(res["o_fine"][..., p.row_src < 0, :] == 0)


def test_fine_sparse_rows_match_restricted_dense():
    prefix, grid, tile = (40, 70), (8, 8, 8), (4, 4, 4)
    p = O.plan(prefix, grid, tile)
    _, tiles, _, _ = coord_rows(prefix, grid, tile)
    rng = np.random.default_rng(5)
    q, k, v, g = (rng.standard_normal((1, 2, p.n_tokens, 16)) for _ in range(4))
    kk = 3
    res = O.layer(q, k, v, g, p, kk, scale=0.25)
    of = O.unpermute(res["o_fine"], p)
    # prefix queries: dense over every token
    n_prefix_tok = sum(prefix)
    dense = _natural_dense(q, k, v, 0.25)
    np.testing.assert_allclose(of[:, :, :n_prefix_tok], dense[:, :, :n_prefix_tok], rtol=1e-11, atol=1e-12)
    # video queries: dense over the tokens of (prefix tiles + kept tiles) only
    for h in range(2):
        for n in range(n_prefix_tok, p.n_tokens, 7):
            i = tiles[n]
            allowed = set(range(p.n_prefix_tiles)) | set(res["topk"][0, h, i - p.n_prefix_tiles].tolist())
            keys = np.array([m for m in range(p.n_tokens) if tiles[m] in allowed])
            want = sdpa64(q[0, h, n:n + 1], k[0, h, keys], v[0, h, keys], 0.25)
            np.testing.assert_allclose(of[0, h, n:n + 1], want, rtol=1e-11, atol=1e-12)


def test_fine_closed_forms():
    p = O.plan((), (4, 4, 8), (4, 4, 4))               # two video tiles, no prefix
    D = 4
    q = np.zeros((p.n_padded, D)); k = np.zeros((p.n_padded, D))
    v = np.tile(np.array([1.5, -2.0, 0.25, 3.0]), (p.n_padded, 1))
    o, lse = O.fine_tile(q, k, v, p, 0, [0, 1], 1.0)
    np.testing.assert_allclose(o, np.broadcast_to(v[:64], o.shape), rtol=1e-15)   # constant V
    np.testing.assert_allclose(lse, math.log(128), rtol=1e-15)                       # 128 equal scores
    # two keys with logits 0 and ln 3 -> weights 1/4, 3/4
    p1 = O.plan((1, 1), (0, 1, 1), (4, 4, 4))
    q1 = np.zeros((p1.n_padded, 2)); q1[0] = [1.0, 0.0]
    k1 = np.zeros((p1.n_padded, 2)); k1[64] = [math.log(3.0), 0.0]
    v1 = np.zeros((p1.n_padded, 2)); v1[0] = [4.0, 0.0]; v1[64] = [0.0, 8.0]
    o1, _ = O.fine_tile(q1, k1, v1, p1, 0, [0, 1], 1.0)
    np.testing.assert_allclose(o1[0], [1.0, 6.0], rtol=1e-14)


# --------------------------------------------------------------------------
# Combine
# --------------------------------------------------------------------------

def test_combine_limits():
    p = O.plan((3,), (4, 4, 4), (4, 4, 4))
    rng = np.random.default_rng(6)
    of = O.permute(rng.standard_normal((1, 1, p.n_tokens, 4)), p)
    oc = rng.standard_normal((1, 1, p.n_tiles, 4))
    tile_of_row = np.repeat(np.arange(p.n_tiles), p.R)
    live = p.row_src >= 0
    out = O.gate_combine(of, np.full(of.shape, -800.0), oc, p)
    np.testing.assert_array_equal(out, of)
    out = O.gate_combine(of, np.zeros(of.shape), oc, p)
    np.testing.assert_allclose(out[..., live, :], (of + 0.5 * oc[..., tile_of_row, :])[..., live, :], rtol=1e-15)
    out = O.gate_combine(of, np.full(of.shape, 800.0), oc, p)
    np.testing.assert_allclose(out[..., live, :], (of + oc[..., tile_of_row, :])[..., live, :], rtol=1e-15)
    assert np.all(out[..., ~live, :] == 0)
    # sigmoid(ln 3) = 3/4
    out = O.gate_combine(of, np.full(of.shape, math.log(3.0)), oc, p)
    np.testing.assert_allclose(out[..., live, :], (of + 0.75 * oc[..., tile_of_row, :])[..., live, :], rtol=1e-14)


def test_projection_closed_forms():
    """The head projection against values fixed without its formula: a hand
    computed 2x2 case, identity weights (y is x's columns split into heads),
    a one-hot permutation of the output features (catches a transposed
    operand or a head/dim mix-up), and sigmoid(0) = 1/2."""
    y = O.project(np.array([[[1.0, 2.0]]]), np.array([[3.0, 4.0], [5.0, 6.0]]), 1, 2)
    np.testing.assert_array_equal(y, [[[[11.0, 17.0]]]])          # [B=1, H=1, N=1, D=2]
    rng = np.random.default_rng(8)
    H, D, B, N = 3, 4, 2, 5
    x = rng.standard_normal((B, N, H * D))
    y = O.project(x, np.eye(H * D), H, D)
    for h in range(H):
        np.testing.assert_array_equal(y[:, h], x[:, :, h * D:(h + 1) * D])
    perm = rng.permutation(H * D)
    y = O.project(x, np.eye(H * D)[perm], H, D)                     # row f of W picks column perm[f]
    for h in range(H):
        for d in range(D):
            np.testing.assert_array_equal(y[:, h, :, d], x[:, :, perm[h * D + d]])
    y = O.project(x, np.zeros((H * D, H * D)), H, D, act="sigmoid")
    assert np.all(y == 0.5)


# --------------------------------------------------------------------------
# Planted mistakes: each must make one of the pins above fail.
# --------------------------------------------------------------------------

def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_planted_mistakes_are_caught(monkeypatch):
    import oracle.vsa_oracle as V

    # 1. prefix segments share tiles (no new tile per segment) -> tile counts move
    orig_plan = V.plan
    def merged_plan(prefix_lens, grid, tile):
        return orig_plan([sum(prefix_lens)] if len(prefix_lens) else [], grid, tile)
    monkeypatch.setattr(O, "plan", merged_plan)
    assert _fails(test_plan_reproduces_worked_example)
    monkeypatch.setattr(O, "plan", orig_plan)

    # 2. transposed coarse scores (k . q instead of q . k)
    orig_coarse = V.coarse_attention
    def transposed(qbar, kbar, vbar, scale):
        s = scale * (kbar @ np.swapaxes(qbar, -1, -2))
        e = np.exp(s - s.max(axis=-1, keepdims=True))
        return s, (e / e.sum(axis=-1, keepdims=True)) @ vbar
    monkeypatch.setattr(O, "coarse_attention", transposed)
    assert _fails(test_coarse_matches_library_attention)
    monkeypatch.setattr(O, "coarse_attention", orig_coarse)

    # 3. ties broken towards the higher tile index
    orig_sel = V.select_topk
    monkeypatch.setattr(O, "select_topk", _high_tie_select)
    assert _fails(lambda: test_topk_matches_brute_force_with_ties(0))
    monkeypatch.setattr(O, "select_topk", orig_sel)

    # 4. sigmoid with the wrong sign
    monkeypatch.setattr(V, "sigmoid", lambda x: 1.0 / (1.0 + np.exp(x)))
    assert _fails(test_combine_limits)
    monkeypatch.undo()

    # 5. pad rows left in the key set (block_len ignored) -> dense equivalence breaks
    orig_fine_tile = V.fine_tile
    def no_mask(q_t, k_t, v_t, p, i, tiles, scale):
        rows = np.concatenate([j * p.R + np.arange(p.R) for j in tiles])
        q = q_t[i * p.R: i * p.R + p.block_len[i]]
        s = scale * (q @ k_t[rows].T)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        l = e.sum(axis=1, keepdims=True)
        return (e @ v_t[rows]) / l, (s.max(axis=1, keepdims=True) + np.log(l))[:, 0]
    monkeypatch.setattr(V, "fine_tile", no_mask)
    assert _fails(lambda: test_fine_at_full_keep_is_dense_attention((40, 70), (4, 8, 8), (4, 4, 4)))
    monkeypatch.undo()

    # 6'. reference ties broken towards the higher index
    orig_ref = V.select_topk_ref
    def high_tie_ref(s, p, k_ref):
        n_p, T = p.n_prefix_tiles, p.n_tiles
        out = np.zeros(s.shape[:-2] + (T - n_p, k_ref), dtype=np.int64)
        cand = np.arange(n_p)
        for idx in np.ndindex(*s.shape[:-2]):
            for i in range(n_p, T):
                order = np.lexsort((-cand, -s[idx + (i,)][:n_p]))
                out[idx + (i - n_p,)] = np.sort(cand[order[:k_ref]])
        return out
    monkeypatch.setattr(O, "select_topk_ref", high_tie_ref)
    assert _fails(lambda: test_reference_topk_matches_brute_force_with_ties(0))
    monkeypatch.setattr(O, "select_topk_ref", orig_ref)

    # 6. projection with the weight not transposed (x @ w instead of x @ w^T)
    orig_project = V.project
    def untransposed(x, w, n_heads, head_dim, act=None):
        y = V.as_f64(x) @ V.as_f64(w)
        B, N = y.shape[0], y.shape[1]
        return y.reshape(B, N, n_heads, head_dim).transpose(0, 2, 1, 3)
    monkeypatch.setattr(O, "project", untransposed)
    assert _fails(test_projection_closed_forms)
    # 7. heads and dims swapped in the split
    def swapped(x, w, n_heads, head_dim, act=None):
        y = V.as_f64(x) @ V.as_f64(w).T
        B, N = y.shape[0], y.shape[1]
        return y.reshape(B, N, head_dim, n_heads).transpose(0, 3, 1, 2)
    monkeypatch.setattr(O, "project", swapped)
    assert _fails(test_projection_closed_forms)
    monkeypatch.setattr(O, "project", orig_project)


def _high_tie_select(s, p, k):
    n_p, T = p.n_prefix_tiles, p.n_tiles
    out = np.zeros(s.shape[:-2] + (T - n_p, k), dtype=np.int64)
    cand = np.arange(n_p, T)
    for idx in np.ndindex(*s.shape[:-2]):
        for i in range(n_p, T):
            order = np.lexsort((-cand, -s[idx + (i,)][n_p:]))
            out[idx + (i - n_p,)] = np.sort(cand[order[:k]])
    return out
