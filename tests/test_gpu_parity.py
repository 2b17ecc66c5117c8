"""GPU parity: every step of the CUDA path, called through the C ABI, against
the fp64 oracle on the same seeded bf16 inputs.

* permutation, tile table and kept-tile sets: bit-exact (a top-k row may
  differ only by a legal near-tie swap, NEAR_TIE_REL at the k-th score);
* pooled means and coarse output: fp32 against fp64;
* o_fine and the layer output: max-abs 2e-2 and mean-abs 2e-3 (bf16 in, fp32
  accumulation), the oracle evaluated under the GPU's own selection;
* the full-size workloads in the benchmark's launch configuration, on sampled
  heads and query tiles the oracle computes one by one.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle as O
from tests.parity import MAX_ABS, MEAN_ABS, assert_close, check_topk, check_topk_row, f64
from tile_sparse_video_b200 import vsa
from tile_sparse_video_b200.inputs import REF2VA, SMALL, TINY, VEDA_104K, Workload, make_inputs, sweep_workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda(libvsa):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


_SEEDS = iter(range(9000, 10000, 7))


def _w(name, B, H, D, prefix, grid, tile, keep_tiles=None, sparsity=None):
    return Workload(name, B=B, H=H, D=D, prefix=prefix, grid=grid, tile=tile, keep_tiles=keep_tiles,
                    sparsity=sparsity, values="iid", gate="marginal", gate_width=64, gate_std=0.2,
                    seed_base=next(_SEEDS))


CASES = [
    TINY,
    SMALL,
    _w("ragged64_b2", 2, 2, 128, (5, 0, 64, 65), (5, 6, 7), (4, 4, 4), keep_tiles=3),
    _w("ragged128", 1, 2, 128, (256, 3), (8, 17, 9), (4, 8, 4), sparsity=0.9),
    _w("d64_r128", 1, 3, 64, (100,), (8, 16, 8), (4, 8, 4), keep_tiles=5),
    _w("noprefix", 1, 2, 128, (), (8, 8, 8), (4, 4, 4), keep_tiles=3),
    _w("keep_all", 1, 2, 64, (40, 70), (4, 8, 8), (4, 4, 4), sparsity=0.0),
    _w("keep_none", 1, 2, 128, (40, 70), (4, 8, 8), (4, 4, 4), keep_tiles=0),
    _w("one_video_tile", 1, 1, 128, (64,), (4, 4, 4), (4, 4, 4), keep_tiles=1),
    _w("prefix_only", 1, 2, 128, (100, 28), (0, 0, 0), (4, 4, 4), keep_tiles=0),
    # 128-row tiles with long kept-tile lists (250 of 300 video tiles)
    _w("wide_k_r128", 1, 1, 128, (256,), (24, 40, 40), (4, 8, 4), keep_tiles=250),
]
# sweep shapes that the oracle finishes quickly (shortest clips, both families)
CASES += [w for w in sweep_workloads() if w.grid[0] == 16 and ("s90" in w.name or "k24" in w.name)
          and w.grid[1] == 32]


def _keep(plan, w):
    return plan.keep_count(keep_ratio=w.keep_ratio, keep_tiles=w.keep_tiles)


def _run(w: Workload, inp=None):
    """The unfused chain (every intermediate visible), plus the fused
    attention + combine entry point on the same inputs."""
    inp = make_inputs(w) if inp is None else inp
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    k = _keep(plan, w)
    q, kk, v, g = (inp[x].cuda() for x in "qkvg")
    layer = vsa.Layer(plan, w.B, w.H, w.D, k, fused=False)
    out = layer(q, kk, v, g)
    _, _, scores, _ = vsa.vsa_coarse_topk(plan, layer.q_t, layer.k_t, layer.v_t, k, want_scores=True)
    _, lse = vsa.vsa_sparse_attn(plan, layer.q_t, layer.k_t, layer.v_t, layer.topk_idx, k, want_lse=True)
    out_t = vsa.vsa_gate_combine(plan, layer.o_fine_t, layer.g_t, layer.o_coarse, natural=False)
    fused, lse_f = vsa.vsa_sparse_attn_combine(plan, layer.q_t, layer.k_t, layer.v_t, layer.topk_idx, k,
                                               g, layer.o_coarse, want_lse=True)
    # the fused permute + pool pass, and coarse + top-k from its pooled means
    ws2 = torch.empty_like(layer.ws)
    slots = vsa.pooled_slots(plan, ws2, w.B, w.H, w.D)
    for x, x_t, pooled in zip((q, kk, v), (layer.q_t, layer.k_t, layer.v_t), slots):
        x_t2, _ = vsa.vsa_permute_pool(plan, x, pooled=pooled)
        assert torch.equal(x_t2, x_t)
    oc2, idx2, _ = vsa.vsa_coarse_topk_pooled(plan, w.B, w.H, w.D, k, ws2)
    vsa.vsa_sync_status(plan)
    assert torch.equal(lse_f, lse)
    layer.fused_out = fused
    layer.pp = (slots, oc2, idx2)
    return inp, plan, k, layer, out, scores, lse, out_t


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_layer_parity(w):
    _check_layer(w, make_inputs(w))


def _growing_logits(w: Workload):
    """Inputs whose key rows grow with their key tile: K of tile j is scaled by
    1 + 3j, so the row maximum of the scores jumps by more than 2^8 from tile
    to tile and the attention kernel's running (reference) max moves, with the
    O rescale that goes with it, on most tiles of every item.  The attention
    is then nearly one-hot, so V is scaled by 1/4 to keep the outputs at the
    unit scale the tolerance is stated for (the moving max does not depend
    on V)."""
    inp = make_inputs(w)
    p = O.plan(w.prefix, w.grid, w.tile)
    tile_of_token = torch.from_numpy(p.untile // p.R)
    c = (1.0 + 3.0 * tile_of_token.double()).view(1, 1, -1, 1)
    inp["k"] = (inp["k"].double() * c).to(torch.bfloat16)
    inp["v"] = (inp["v"].double() * 0.25).to(torch.bfloat16)
    return inp


@pytest.mark.parametrize("w", [
    _w("growing_logits_r64", 1, 2, 128, (100, 28), (8, 8, 8), (4, 4, 4), keep_tiles=5),
    _w("growing_logits_r128", 1, 2, 128, (256,), (8, 16, 8), (4, 8, 4), keep_tiles=3),
], ids=lambda w: w.name)
def test_layer_parity_moving_max(w):
    _check_layer(w, _growing_logits(w))


def _check_layer(w: Workload, inp):
    inp, plan, k, layer, out, scores, lse, out_t = _run(w, inp)
    p = O.plan(w.prefix, w.grid, w.tile)
    gpu_idx = layer.topk_idx.cpu().numpy().astype(np.int64)
    ref = O.layer(*(inp[x] for x in "qkvg"), p, k, kept=gpu_idx)

    # step 1: permutation, bit-exact (pad rows zero)
    for name in ("q_t", "k_t", "v_t", "g_t"):
        assert np.array_equal(f64(getattr(layer, name)), ref[name]), name
    # step 2: pooled means (workspace layout of the header) and coarse output
    T, D, BH = p.n_tiles, w.D, w.B * w.H
    pooled = layer.ws[: 3 * BH * T * D * 4].view(torch.float32).view(3, w.B, w.H, T, D)
    for i, name in enumerate(("qbar", "kbar", "vbar")):
        np.testing.assert_allclose(f64(pooled[i]), ref[name], rtol=1e-5, atol=1e-6, err_msg=name)
    np.testing.assert_allclose(f64(layer.o_coarse), ref["o_coarse"], rtol=1e-4, atol=1e-5)
    slots, oc2, idx2 = layer.pp
    for i, name in enumerate(("qbar", "kbar", "vbar")):
        np.testing.assert_allclose(f64(slots[i]), ref[name], rtol=1e-5, atol=1e-6, err_msg=name + " (fused)")
    np.testing.assert_allclose(f64(oc2), ref["o_coarse"], rtol=1e-4, atol=1e-5)
    # step 3: selection, bit-exact up to legal near-tie swaps
    near = check_topk(gpu_idx, ref["scores"], p, k)
    assert near <= max(1, int(np.prod(gpu_idx.shape[:-1])) // 50)
    near2 = check_topk(idx2.cpu().numpy().astype(np.int64), ref["scores"], p, k)
    assert near2 <= max(1, int(np.prod(gpu_idx.shape[:-1])) // 50)
    if k > 0:
        gs = f64(scores)
        want = np.take_along_axis(ref["scores"][..., p.n_prefix_tiles:, :], gpu_idx, axis=-1)
        np.testing.assert_allclose(gs, want, rtol=1e-4, atol=1e-5)
    # step 4: fine attention under the GPU's selection
    assert_close(f64(layer.o_fine_t), ref["o_fine"], what="o_fine")
    live = p.row_src >= 0
    np.testing.assert_allclose(f64(lse)[..., live], ref["lse"][..., live], atol=2e-3)
    assert np.all(f64(lse)[..., ~live] == 0)
    # step 5: combine, both output layouts, and the fused attention + combine
    assert_close(f64(out), ref["out"], what="out")
    assert_close(f64(layer.fused_out), ref["out"], what="fused out")
    assert_close(f64(out_t), ref["out_t"], what="out_t")
    assert np.all(f64(out_t)[..., ~live, :] == 0)
    assert torch.equal(vsa.vsa_unpermute(plan, out_t), out)


@pytest.mark.parametrize("law", ["three_keys", "one_key", "quantised"])
def test_topk_heavy_ties(law):
    """Selections whose k-th score sits among many equal scores, against the
    oracle's (score descending, index ascending) order, which is unique here,
    so the kept tiles must match exactly.  three_keys: every pooled key is one
    of three vectors (about 50 equal scores per value in a row of 153 key
    tiles, more than the range histogram's 32-candidate bin, so the exact
    radix select decides); one_key: every score of a row equal (a zero range);
    quantised: one-hot pooled queries against keys on an 1/8 grid (8 distinct
    scores per row, the candidate ranking inside one histogram bin decides
    among equal scores).  Equal pooled keys give equal fp32 and fp64 scores,
    and distinct grid values stay ordered, so rounding cannot move a tie."""
    w = SMALL
    B, H, D = 1, 2, w.D
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    p = O.plan(w.prefix, w.grid, w.tile)
    T = p.n_tiles
    k = plan.keep_count(keep_tiles=40)
    g = torch.Generator().manual_seed(4242)
    q = torch.randn(B, H, T, D, generator=g)
    v = torch.randn(B, H, T, D, generator=g)
    if law == "three_keys":
        kk = torch.randn(3, D, generator=g)[torch.randint(0, 3, (B, H, T), generator=g)]
    elif law == "one_key":
        kk = torch.randn(D, generator=g).expand(B, H, T, D).contiguous()
    else:
        q = torch.zeros(B, H, T, D)
        q[..., 0] = 1.0
        kk = torch.randn(B, H, T, D, generator=g)
        kk[..., 0] = torch.randint(0, 8, (B, H, T), generator=g).float() / 8
    ws = torch.zeros(plan.workspace_size(B, H, D, k), dtype=torch.uint8, device="cuda")
    for slot, x in zip(vsa.pooled_slots(plan, ws, B, H, D), (q, kk, v)):
        slot.copy_(x.cuda())
    oc, idx, _ = vsa.vsa_coarse_topk_pooled(plan, B, H, D, k, ws)
    s, oc_ref = O.coarse_attention(q.double().numpy(), kk.double().numpy(), v.double().numpy(), D ** -0.5)
    assert np.array_equal(idx.cpu().numpy().astype(np.int64), O.select_topk(s, p, k))
    np.testing.assert_allclose(f64(oc), oc_ref, rtol=1e-4, atol=1e-5)
    vsa.vsa_sync_status(plan)


def test_topk_non_finite_scores_stay_valid():
    """Pooled means holding NaN and +-inf (whole key rows of NaN, keys with
    infinite entries, a query row of NaN): the selection is still k distinct
    video tile indices per row in ascending order, nothing is recorded in the
    status word, and rows without a non-finite score match the oracle.  A NaN
    score ranks by its order key (the exact radix select), so the keep pass
    never selects more than k."""
    w = SMALL
    B, H, D = 1, 2, w.D
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    p = O.plan(w.prefix, w.grid, w.tile)
    T, n_p = p.n_tiles, p.n_prefix_tiles
    k = plan.keep_count(keep_tiles=40)
    g = torch.Generator().manual_seed(515)
    q = torch.randn(B, H, T, D, generator=g)
    kk = torch.randn(B, H, T, D, generator=g)
    v = torch.randn(B, H, T, D, generator=g)
    # head 0: a NaN key row, keys with +-inf entries (+-inf or NaN scores);
    # head 1: one NaN query row, every other row finite
    kk[0, 0, n_p + 3] = float("nan")
    kk[0, 0, n_p + 10, 5] = float("inf")
    kk[0, 0, n_p + 7, 0] = float("-inf")
    kk[0, 0, n_p + 9, 1] = float("inf")
    kk[0, 0, n_p + 9, 2] = float("-inf")
    q[0, 1, n_p + 20] = float("nan")
    ws = torch.zeros(plan.workspace_size(B, H, D, k), dtype=torch.uint8, device="cuda")
    for slot, x in zip(vsa.pooled_slots(plan, ws, B, H, D), (q, kk, v)):
        slot.copy_(x.cuda())
    _, idx, _ = vsa.vsa_coarse_topk_pooled(plan, B, H, D, k, ws)
    vsa.vsa_sync_status(plan)
    got = idx.cpu().numpy().astype(np.int64)
    assert np.all(np.diff(got, axis=-1) > 0) and got.min() >= n_p and got.max() < T
    with np.errstate(invalid="ignore", over="ignore"):
        s, _ = O.coarse_attention(q.double().numpy(), kk.double().numpy(), v.double().numpy(), D ** -0.5)
    checked = 0
    for h in range(H):
        for i in range(n_p, T):
            row = s[0, h, i]
            if np.all(np.isfinite(row[n_p:])):
                check_topk_row(got[0, h, i - n_p], row, n_p, k)
                checked += 1
    assert checked == T - n_p - 1        # head 1 without its NaN query row


def test_keep_all_equals_dense_attention():
    """k = every video tile: the fine output is plain dense attention over all
    real tokens (torch's own routine, fp32 on the GPU)."""
    w = _w("dense_check", 1, 2, 128, (40, 70), (4, 8, 8), (4, 4, 4), sparsity=0.0)
    inp, plan, k, layer, *_ = _run(w)      # unfused layer: o_fine_t is kept
    assert k == plan.n_video_tiles
    o_nat = vsa.vsa_unpermute(plan, layer.o_fine_t)
    q, kk, v = (inp[x].cuda().float() for x in "qkv")
    dense = torch.nn.functional.scaled_dot_product_attention(q, kk, v, scale=w.D ** -0.5)
    assert_close(f64(o_nat), f64(dense), what="dense")


def _sampled(w: Workload, heads, n_video_samples, seed):
    inp = make_inputs(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    k = _keep(plan, w)
    dev = torch.device("cuda")
    q, kk, v, g = (inp[x].to(dev) for x in "qkvg")
    layer = vsa.Layer(plan, w.B, w.H, w.D, k)          # the fused chain the benchmark times
    out = layer(q, kk, v, g)
    o_fine_t, _ = vsa.vsa_sparse_attn(plan, layer.q_t, layer.k_t, layer.v_t, layer.topk_idx, k)
    vsa.vsa_sync_status(plan)
    p = O.plan(w.prefix, w.grid, w.tile)
    rng = np.random.default_rng(seed)
    scale = w.D ** -0.5
    n_near = 0
    for b in range(w.B):
        for h in heads:
            q_t, k_t, v_t, g_t = (O.permute(inp[x][b, h].to(torch.float64).numpy(), p) for x in "qkvg")
            qb, kb, vb = O.pool(q_t, p), O.pool(k_t, p), O.pool(v_t, p)
            s, oc = O.coarse_attention(qb, kb, vb, scale)
            np.testing.assert_allclose(f64(layer.o_coarse[b, h]), oc, rtol=1e-4, atol=1e-5)
            idx = layer.topk_idx[b, h].cpu().numpy().astype(np.int64)
            for r in range(p.n_video_tiles):
                n_near += check_topk_row(idx[r], s[p.n_prefix_tiles + r], p.n_prefix_tiles, k)
            tiles = list(range(p.n_prefix_tiles)) + list(
                p.n_prefix_tiles + rng.choice(p.n_video_tiles, n_video_samples, replace=False))
            tiles.append(p.n_tiles - 1)
            out_bh = out[b, h].cpu()
            o_fine_bh = o_fine_t[b, h].cpu()
            for i in sorted(set(tiles)):
                kept = idx[i - p.n_prefix_tiles] if i >= p.n_prefix_tiles else None
                o, _ = O.fine_tile(q_t, k_t, v_t, p, i, O.key_tiles(p, i, kept), scale)
                r0, r1 = i * p.R, i * p.R + int(p.block_len[i])
                want = o + O.sigmoid(g_t[r0:r1]) * oc[i]
                tok = torch.from_numpy(p.row_src[r0:r1])
                # o_fine and out are linear in V: the tolerance (stated for unit-scale
                # values) scales with the head's value scale s_h where it exceeds 1
                sv = max(1.0, float(inp["value_scale"][b, h]))
                assert_close(f64(o_fine_bh[r0:r1]), o, MAX_ABS * sv, MEAN_ABS * sv, what=f"o_fine h{h} tile{i}")
                assert_close(f64(out_bh[tok]), want, MAX_ABS * sv, MEAN_ABS * sv, what=f"out h{h} tile{i}")
    assert n_near <= max(2, w.B * len(heads) * p.n_video_tiles // 50)


# the reference-to-video family of the sweep at its shortest clip (24 x 42
# grid: partial w-cubes; six-segment prefix; B = 2), at 75 % and at k = 24
REF2VA_SWEEP = [w for w in sweep_workloads()
                if w.grid[:2] == (16, 24) and (w.name.endswith("_s75_b2") or "_k24_" in w.name)]


@pytest.mark.parametrize("w", REF2VA_SWEEP, ids=lambda w: w.name)
def test_ref2va_sweep_sampled(w):
    _sampled(w, (0, 29, 41), 12, seed=5)


@pytest.mark.parametrize("w,heads,n", [(REF2VA, (0, 17, 41), 24), (VEDA_104K, (0, 23, 41), 16),
                                       (replace(VEDA_104K, name="veda_h56", H=56), (0, 55), 8)],
                         ids=["ref2va_full", "veda_104k_full", "veda_h56_full"])
def test_full_size_sampled(w, heads, n):
    _sampled(w, heads, n, seed=11)


def test_error_paths():
    w = TINY
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    x = torch.zeros(1, 2, plan.n_tokens * 64 + 8, dtype=torch.bfloat16, device="cuda")
    mis = x.view(-1)[1:1 + 2 * plan.n_tokens * 64].view(1, 2, plan.n_tokens, 64)
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_permute(plan, mis)
    assert e.value.status == 1
    q_t = torch.zeros(1, 2, plan.n_padded, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_coarse_topk(plan, q_t, q_t, q_t, 2, ws=ws)
    assert e.value.status == 4
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_coarse_topk(plan, q_t, q_t, q_t, plan.n_video_tiles + 1)
    assert e.value.status == 1
    bad = torch.zeros(1, 2, plan.n_padded, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_permute(plan, torch.zeros(1, 2, plan.n_tokens, 96, dtype=torch.bfloat16, device="cuda"), bad)
    assert e.value.status == 2
    vsa.vsa_sync_status(plan)


def test_bad_kept_index_is_reported():
    """An out-of-range kept-tile index is clamped by the kernel and reported
    through the status word (no fault, no hang)."""
    w = TINY
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    t = torch.randn(1, 2, plan.n_padded, 64, device="cuda").to(torch.bfloat16)
    idx = torch.full((1, 2, plan.n_video_tiles, 2), plan.n_prefix_tiles, dtype=torch.int32, device="cuda")
    idx[0, 1, 2, 1] = plan.n_tiles + 5
    vsa.vsa_sparse_attn(plan, t, t, t, idx, 2)
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_sync_status(plan)
    assert e.value.status == 7
    vsa.vsa_sync_status(plan)       # cleared


def test_bounded_wait_gives_up_and_reports():
    """The bounded device wait every kernel uses, on an mbarrier nothing
    completes (vsa_check_bounded_wait): both waiters give up within the bound,
    the timeout is reported through the status word, and the context still
    runs a layer correctly afterwards."""
    import time
    w = TINY
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    t0 = time.perf_counter()
    res = vsa.vsa_check_bounded_wait(plan)
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_sync_status(plan)
    elapsed = time.perf_counter() - t0
    assert e.value.status == 6                  # VSA_ERR_DEVICE_TIMEOUT
    assert res.cpu().tolist() == [0, 0]          # both waits gave up
    assert 1.5 < elapsed < 30.0, elapsed         # the 2 s bound, not a hang
    vsa.vsa_sync_status(plan)                    # cleared
    _check_layer(w, make_inputs(w))              # the context is still usable


@pytest.mark.parametrize("w", [
    TINY,                                                                  # 64-row tiles (pairs)
    _w("abort_r128", 1, 2, 128, (256,), (8, 16, 8), (4, 8, 4), keep_tiles=3),
], ids=lambda w: w.name)
def test_attention_abort_path(w):
    """The attention kernels' own failure path, run on the GPU without a
    fault: with their wait bound cut to 100 ns (vsa_debug_set_wait_limit) the
    forward kernel's and the backward kernels' waits run out, each records
    VSA_ERR_DEVICE_TIMEOUT, drains its TMA loads and MMAs, frees its tensor
    memory and returns well within a second; with the bound restored the same
    context runs the layer, forward and backward, correctly."""
    import time
    inp = make_inputs(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    k = _keep(plan, w)
    q, kk, v, g = (inp[x].cuda() for x in "qkvg")
    train = vsa.TrainingLayer(plan, w.B, w.H, w.D, k)
    train.forward(q, kk, v, g)
    d_out = torch.randn(train.out.shape, device="cuda").to(torch.bfloat16)
    vsa.vsa_sync_status(plan)
    try:
        vsa.vsa_debug_set_wait_limit(100)
        for what in ("forward", "backward"):
            timed_out = False
            for _ in range(5):             # a wait that happened to finish in time: try again
                t0 = time.perf_counter()
                if what == "forward":
                    vsa.vsa_sparse_attn(plan, train.q_t, train.k_t, train.v_t, train.topk_idx, k)
                else:
                    train.backward(d_out)
                try:
                    vsa.vsa_sync_status(plan)
                except vsa.VsaError as e:
                    assert e.status == 6, e              # VSA_ERR_DEVICE_TIMEOUT
                    timed_out = True
                elapsed = time.perf_counter() - t0
                assert elapsed < 1.0, (what, elapsed)
                if timed_out:
                    break
            assert timed_out, f"the {what} kernels never gave up under a 100 ns bound"
    finally:
        vsa.vsa_debug_set_wait_limit(0)
    vsa.vsa_sync_status(plan)
    _check_layer(w, inp)
    grads = train.backward(d_out)
    vsa.vsa_sync_status(plan)
    assert all(torch.isfinite(x.float()).all() for x in grads)


def test_empty_batch_is_a_no_op():
    plan = vsa.Plan(TINY.prefix, TINY.grid, TINY.tile)
    x = torch.empty(0, 2, plan.n_tokens, 64, dtype=torch.bfloat16, device="cuda")
    assert vsa.vsa_permute(plan, x).shape == (0, 2, plan.n_padded, 64)
    vsa.vsa_sync_status(plan)


def test_layer_pipeline_matches_layer():
    """The library's runner behind vsa.LayerPipeline (copy-in, compute and
    copy-out of consecutive layers overlapped on three streams, two buffer
    sets) gives bit-identical outputs to calling the Layer once per input set,
    for more layers than buffer sets, and again on a second run of the same
    runner."""
    from dataclasses import replace
    w = SMALL
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    k = _keep(plan, w)
    sets = [make_inputs(replace(w, seed_base=w.seed_base + 31 * i)) for i in range(5)]
    host = [{n: s[n].pin_memory() for n in "qkvg"} for s in sets]
    pipe = vsa.LayerPipeline(plan, w.B, w.H, w.D, k)
    layer = vsa.Layer(plan, w.B, w.H, w.D, k)
    wants = [layer(*(s[n].cuda() for n in "qkvg")).cpu() for s in sets]
    for order in (range(5), (4, 2, 0)):
        outs = [torch.empty(w.B, w.H, plan.n_tokens, w.D, dtype=torch.bfloat16).pin_memory()
                for _ in order]
        pipe.run([host[i] for i in order], outs)
        torch.cuda.synchronize()
        assert pipe.elapsed_ms() > 0
        for i, got in zip(order, outs):
            assert torch.equal(got, wants[i])
    pipe.close()
    vsa.vsa_sync_status(plan)


def test_runner_rejects_bad_host_tensors():
    w = TINY
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    k = _keep(plan, w)
    pipe = vsa.LayerPipeline(plan, w.B, w.H, w.D, k)
    good = torch.zeros(w.B, w.H, plan.n_tokens, w.D, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pipe.run([{n: good for n in "qkvg"}], [good.float()])
    with pytest.raises(ValueError):
        pipe.run([{n: good for n in "qkvg"}], [])
    with pytest.raises(vsa.VsaError):
        vsa.LayerPipeline(plan, w.B, w.H, 96, k)
    pipe.close()


REF_CASES = [
    (SMALL, 3),                                                    # 25 reference tiles -> 3
    (SMALL, 0),                                                    # no reference tile kept
    (_w("ref_r128", 1, 2, 128, (256, 200, 60), (8, 16, 8), (4, 8, 4), keep_tiles=3), 1),
    (_w("ref_d64_b2", 2, 2, 64, (64, 64, 64, 30), (4, 8, 8), (4, 4, 4), sparsity=0.75), 2),
]


@pytest.mark.parametrize("w,k_ref", REF_CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_reference_thinning_parity(w, k_ref):
    """Reference tiles thinned to each video query tile's top k_ref (the Veda
    reference_sparsity reading): the reference selection against the oracle's
    fp64 ranking (bit-exact up to legal near-ties), and o_fine, the unfused and
    the fused outputs against the oracle under the GPU's selections."""
    inp = make_inputs(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    k = _keep(plan, w)
    q, kk, v, g = (inp[x].cuda() for x in "qkvg")
    layer = vsa.Layer(plan, w.B, w.H, w.D, k, fused=False, k_ref=k_ref)
    out = layer(q, kk, v, g)
    fused = vsa.Layer(plan, w.B, w.H, w.D, k, k_ref=k_ref)
    out_f = fused(q, kk, v, g)
    vsa.vsa_sync_status(plan)
    p = O.plan(w.prefix, w.grid, w.tile)
    gpu_idx = layer.topk_idx.cpu().numpy().astype(np.int64)
    gpu_ref = layer.topk_ref.cpu().numpy().astype(np.int64)
    assert torch.equal(layer.topk_ref, fused.topk_ref)
    ref = O.layer(*(inp[x] for x in "qkvg"), p, k, kept=gpu_idx, kept_ref=gpu_ref)
    n_near = 0
    for idx in np.ndindex(*gpu_ref.shape[:-2]):
        for r in range(gpu_ref.shape[-2]):
            row = ref["scores"][idx + (p.n_prefix_tiles + r,)][:p.n_prefix_tiles]
            n_near += check_topk_row(gpu_ref[idx + (r,)], row, 0, k_ref)
    assert n_near <= max(1, int(np.prod(gpu_ref.shape[:-1])) // 50)
    assert_close(f64(layer.o_fine_t), ref["o_fine"], what="o_fine")
    assert_close(f64(out), ref["out"], what="out")
    assert_close(f64(out_f), ref["out"], what="fused out")


def test_reference_thinning_keep_all_is_unthinned():
    """k_ref = n_p through the thinned path (selection list of every reference
    tile in order) gives the unthinned layer's output bit for bit."""
    w = SMALL
    inp = make_inputs(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    k = _keep(plan, w)
    q, kk, v, g = (inp[x].cuda() for x in "qkvg")
    thin = vsa.Layer(plan, w.B, w.H, w.D, k, k_ref=plan.n_prefix_tiles)
    base = vsa.Layer(plan, w.B, w.H, w.D, k)
    assert torch.equal(thin(q, kk, v, g), base(q, kk, v, g))
    want = torch.arange(plan.n_prefix_tiles, dtype=torch.int32, device="cuda")
    assert torch.equal(thin.topk_ref, want.expand_as(thin.topk_ref))
    assert vsa.vsa_keep_count_ref(plan, keep_ratio=0.1) == 3
    vsa.vsa_sync_status(plan)
