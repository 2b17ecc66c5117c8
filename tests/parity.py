"""Comparison helpers for the GPU-vs-oracle parity tests (no arithmetic of the
layer lives here: only tolerances, the near-tie acceptance rule and
bookkeeping)."""
import numpy as np
import torch

import oracle as O

# Output tolerance for bf16 inputs with fp32 accumulation.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# The same error measured against the bf16 floor (the oracle's own values
# rounded to bf16, see bf16_floor): a bf16 output cannot do better than the
# floor, and P rounded to bf16 before the PV product adds a comparable share.
# Every forward comparison must stay within these multiples of its floor,
# whatever the magnitude of its values (the head-scaled workloads included).
FLOOR_MAX_MULT = 5.0
FLOOR_MEAN_MULT = 3.0
# Near-tie rule for the top-k boundary: scores within this relative gap may
# swap.
NEAR_TIE_REL = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


# Every output comparison, with its bf16 floor: (what, max err, mean err,
# max floor, mean floor).  The floor is the error of the oracle itself once
# rounded to bf16 (|bf16(want) - want|), the least any bf16 output can have.
RECORDS = []
CURRENT_TEST = [""]          # set per test by the conftest fixture


def bf16_floor(want):
    """Max and mean of |bf16(want) - want| (round to nearest even)."""
    w = torch.from_numpy(np.ascontiguousarray(want, dtype=np.float64))
    f = (w.to(torch.bfloat16).to(torch.float64) - w).abs()
    return (float(f.max()), float(f.mean())) if f.numel() else (0.0, 0.0)


def assert_close(got, want, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what="", floor_mult=True):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - want)
    mx, mn = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    fmx, fmn = bf16_floor(want)
    RECORDS.append((f"{CURRENT_TEST[0]}: {what}", mx, mn, fmx, fmn))
    assert mx <= max_abs and mn <= mean_abs, \
        f"{what}: max-abs {mx:.3e}, mean-abs {mn:.3e} (bf16 floor {fmx:.3e} / {fmn:.3e})"
    if floor_mult:
        assert mx <= FLOOR_MAX_MULT * fmx + 1e-30 and mn <= FLOOR_MEAN_MULT * fmn + 1e-30, \
            (f"{what}: max-abs {mx:.3e}, mean-abs {mn:.3e} above {FLOOR_MAX_MULT} / "
             f"{FLOOR_MEAN_MULT} x the bf16 floor {fmx:.3e} / {fmn:.3e}")
    return mx, mn


def check_topk_row(sel, scores_row, n_p, k):
    """Validate one row of the GPU selection against fp64 oracle scores.

    sel: k global tile indices (GPU); scores_row: fp64 scores over all T tiles.
    Returns 0 when sel equals the oracle's exact choice, 1 for a legal
    near-tie swap; raises AssertionError otherwise."""
    T = scores_row.size
    sel = np.asarray(sel, dtype=np.int64)
    assert sel.size == k
    if k == 0:
        return 0
    assert np.all(np.diff(sel) > 0), "not strictly ascending"
    assert sel.min() >= n_p and sel.max() < T, "index outside the video tiles"
    cand = np.arange(n_p, T)
    s = scores_row[n_p:]
    order = np.lexsort((cand, -s))
    want = np.sort(cand[order[:k]])
    if np.array_equal(sel, want):
        return 0
    s_k = s[order[k - 1]]
    s_k1 = s[order[k]] if k < s.size else s_k
    tol = NEAR_TIE_REL * max(abs(s_k), abs(s_k1), 1e-30)
    extra = np.setdiff1d(sel, want)
    missing = np.setdiff1d(want, sel)
    assert np.all(scores_row[extra] >= s_k - tol), "kept a tile clearly below the k-th score"
    assert np.all(scores_row[missing] <= s_k + tol), "dropped a tile clearly above the k-th score"
    return 1


def check_topk(gpu_idx, scores, p: O.Plan, k):
    """gpu_idx [..., n_v, k]; scores [..., T, T] fp64.  Returns near-tie rows."""
    n = 0
    for idx in np.ndindex(*gpu_idx.shape[:-2]):
        for r in range(gpu_idx.shape[-2]):
            n += check_topk_row(gpu_idx[idx + (r,)], scores[idx + (p.n_prefix_tiles + r,)],
                                p.n_prefix_tiles, k)
    return n
