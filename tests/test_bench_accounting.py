"""The benchmark's work accounting, on the CPU: the algorithmic FLOP and bytes
that the roofline fractions divide by, pinned to brute-force counts over the
oracle's plan and key sets (not to bench.py's own formulas), and the small
helpers around them."""
import os
import sys

import numpy as np
import pytest
import torch

import oracle as O
from tile_sparse_video_b200 import vsa
from tile_sparse_video_b200.inputs import REF2VA, SMALL, TINY, VEDA_104K

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _random_selection(p: O.Plan, k: int, BH: int, seed: int) -> np.ndarray:
    """k distinct ascending video key tiles per (head, video query tile)."""
    rng = np.random.default_rng(seed)
    n_v = p.n_video_tiles
    out = np.empty((BH, n_v, k), np.int64)
    for h in range(BH):
        for i in range(n_v):
            out[h, i] = np.sort(rng.choice(n_v, size=k, replace=False)) + p.n_prefix_tiles
    return out


@pytest.mark.parametrize("w", [TINY, SMALL, REF2VA], ids=lambda w: w.name)
def test_kept_pairs_and_flop_match_brute_force(w):
    p = O.plan(w.prefix, w.grid, w.tile)
    k = O.keep_count(p.n_video_tiles, p.n_prefix_tiles, keep_ratio=w.keep_ratio, keep_tiles=w.keep_tiles)
    acct = bench.geometry_counts(w, p.n_prefix_tiles, p.n_tiles, k)
    sel = _random_selection(p, k, 1, seed=3)
    pairs = sum(len(O.key_tiles(p, i, sel[0, i - p.n_prefix_tiles] if i >= p.n_prefix_tiles else None))
                for i in range(p.n_tiles))
    assert acct["pairs"] == pairs
    BH = w.B * w.H
    assert acct["kept_flop"] == 4.0 * w.D * p.R * p.R * pairs * BH
    assert acct["dense_flop"] == 4.0 * p.n_tokens ** 2 * w.D * BH


@pytest.mark.parametrize("w", [TINY, SMALL], ids=lambda w: w.name)
def test_live_flop_matches_brute_force(w):
    """Live-row work: 4*D*block_len[i]*block_len[j] summed over every head's
    kept (query tile i, key tile j) pairs, the sets taken from the oracle."""
    p = O.plan(w.prefix, w.grid, w.tile)
    plan = vsa.Plan(w.prefix, w.grid, w.tile, device=-1)
    k = O.keep_count(p.n_video_tiles, p.n_prefix_tiles, keep_ratio=w.keep_ratio, keep_tiles=w.keep_tiles)
    BH = w.B * w.H
    sel = _random_selection(p, k, BH, seed=11)
    want = 0.0
    for h in range(BH):
        for i in range(p.n_tiles):
            row = sel[h, i - p.n_prefix_tiles] if i >= p.n_prefix_tiles else None
            for j in O.key_tiles(p, i, row):
                want += 4.0 * w.D * p.block_len[i] * p.block_len[j]
    idx = torch.from_numpy(sel.reshape(w.B, w.H, p.n_video_tiles, k).astype(np.int32))
    assert bench.live_flop(plan, idx, w.D) == pytest.approx(want, rel=1e-12)
    plan.close()


def test_headline_accounting():
    """The 104,704-token layer: 2 prefix + 816 video tiles of 128 rows, k = 82:
    70,180 kept tile pairs per head, 24.73 TFLOP over 42 heads; the bytes the
    permute and the fused attention must move."""
    w = VEDA_104K
    p = O.plan(w.prefix, w.grid, w.tile)
    k = O.keep_count(p.n_video_tiles, p.n_prefix_tiles, keep_ratio=w.keep_ratio, keep_tiles=w.keep_tiles)
    assert (p.n_prefix_tiles, p.n_video_tiles, p.R, k) == (2, 816, 128, 82)
    acct = bench.geometry_counts(w, p.n_prefix_tiles, p.n_tiles, k)
    assert acct["pairs"] == 816 * (2 + 82) + 2 * 818 == 70180
    assert acct["kept_flop"] == pytest.approx(24.727e12, rel=1e-4)
    N, N_pad, BHD2 = 104704, 818 * 128, 42 * 128 * 2
    assert acct["permute_bytes"] == 3 * (N + N_pad) * BHD2            # Q, K, V: read N rows, write N_pad
    assert acct["attn_bytes"] == 3 * N_pad * BHD2 + 2 * N * BHD2      # Q, K, V tiled; gate in, output out
    assert acct["attn_bytes"] == pytest.approx(5.63e9, rel=1e-3)


def test_fp32_peak_and_clock_normalisation():
    assert bench.fp32_core_peak_tflops() == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)
    c = bench.clock_normalised(1000.0, 20.0, {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0})
    assert c["mcycles_per_launch"] == pytest.approx(30.0)
    assert c["achieved_at_max_clock"] == pytest.approx(1310.0)
    assert bench.clock_normalised(1000.0, 20.0, {}) == {"sm_mhz": None}


def test_traffic_digest_ignores_comments_only():
    base = "int f(int a) {\n  return a + 1;  // add one\n}\n"
    assert bench.kernel_source_digest(base) == bench.kernel_source_digest(
        "/* header */ int f(int a) {   return a + 1; }")
    assert bench.kernel_source_digest(base) != bench.kernel_source_digest(base.replace("+ 1", "+ 2"))
