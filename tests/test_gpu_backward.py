"""GPU parity of the backward pass (called through the C ABI) against the fp64
oracle's backward, on the same seeded bf16 inputs and upstream gradient, with
the oracle evaluated under the GPU's own selection (the selection passes no
gradient).

Tolerances, from the arithmetic:
* combine backward: delta is an fp32 sum of D products of bf16 values and
  d_o_coarse an fp32 sum over at most R rows: 1e-4 of the tensor's largest
  magnitude; d_gate is one bf16 rounding (2^-8 relative) of an fp32 product.
* coarse backward: fp32 matrix products over T and D terms: 1e-3 of the
  largest magnitude.
* attention backward and the whole layer: P and dS are rounded to bf16
  (relative 2^-9) before their products, o_fine enters delta as bf16 and the
  outputs are bf16, with fp32 accumulation: max error <= 2e-2 and mean error
  <= 4e-3 of the reference's largest and mean magnitude.
"""
import numpy as np
import pytest
import torch

import oracle as O
from tests.parity import RECORDS, bf16_floor, f64
from tile_sparse_video_b200 import vsa
from tile_sparse_video_b200.inputs import SMALL, TINY, Workload, make_grad_output, make_inputs

pytestmark = pytest.mark.gpu

REL_MAX = 2e-2
REL_MEAN = 4e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda(libvsa):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


_SEEDS = iter(range(12000, 13000, 7))


def _w(name, B, H, D, prefix, grid, tile, keep_tiles=None, sparsity=None):
    return Workload(name, B=B, H=H, D=D, prefix=prefix, grid=grid, tile=tile, keep_tiles=keep_tiles,
                    sparsity=sparsity, values="iid", gate="marginal", gate_width=64, gate_std=0.2,
                    seed_base=next(_SEEDS))


def assert_rel(got, want, rel_max=REL_MAX, rel_mean=REL_MEAN, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    if want.size == 0:
        return
    err = np.abs(got - want)
    fmx, fmn = bf16_floor(want)
    from tests import parity
    RECORDS.append((f"{parity.CURRENT_TEST[0]}: {what}", float(err.max()), float(err.mean()), fmx, fmn))
    scale_max = float(np.abs(want).max())
    scale_mean = float(np.abs(want).mean())
    assert err.max() <= rel_max * scale_max + 1e-30, (
        f"{what}: max err {err.max():.3e} vs {rel_max} x {scale_max:.3e}")
    assert err.mean() <= rel_mean * scale_mean + 1e-30, (
        f"{what}: mean err {err.mean():.3e} vs {rel_mean} x {scale_mean:.3e}")


def _keep(plan, w):
    return plan.keep_count(keep_ratio=w.keep_ratio, keep_tiles=w.keep_tiles)


CASES = [
    (TINY, None),
    (_w("ragged64_b2", 2, 2, 128, (5, 0, 64, 65), (5, 6, 7), (4, 4, 4), keep_tiles=3), None),
    (_w("ragged128", 1, 2, 128, (256, 3), (8, 17, 9), (4, 8, 4), sparsity=0.9), None),
    (_w("d64_r128", 1, 2, 64, (100,), (8, 16, 8), (4, 8, 4), keep_tiles=5), None),
    (_w("noprefix", 1, 2, 128, (), (8, 8, 8), (4, 4, 4), keep_tiles=3), None),
    (_w("keep_all", 1, 2, 64, (40, 70), (4, 8, 8), (4, 4, 4), sparsity=0.0), None),
    (_w("keep_none", 1, 2, 128, (40, 70), (4, 8, 8), (4, 4, 4), keep_tiles=0), None),
    (_w("prefix_only", 1, 2, 128, (100, 28), (0, 0, 0), (4, 4, 4), keep_tiles=0), None),
    (_w("ref_thin_r64", 1, 2, 128, (40, 70, 130), (4, 8, 8), (4, 4, 4), keep_tiles=2), 2),
    (_w("ref_thin_r128", 1, 2, 128, (256, 300), (8, 16, 8), (4, 8, 4), keep_tiles=3), 1),
    (SMALL, None),
]


def _run(w: Workload, k_ref):
    inp = make_inputs(w)
    d_out = make_grad_output(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    k = _keep(plan, w)
    layer = vsa.TrainingLayer(plan, w.B, w.H, w.D, k, k_ref=k_ref)
    out = layer.forward(*(inp[x].cuda() for x in "qkvg"))
    grads = layer.backward(d_out.cuda())
    vsa.vsa_sync_status(plan)
    return inp, d_out, plan, k, layer, out, grads


@pytest.mark.parametrize("w,k_ref", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_layer_backward_parity(w, k_ref):
    inp, d_out, plan, k, layer, out, grads = _run(w, k_ref)
    p = O.plan(w.prefix, w.grid, w.tile)
    sel = layer.topk_idx.cpu().numpy().astype(np.int64)
    sel_ref = None if k_ref is None else layer.topk_ref.cpu().numpy().astype(np.int64)
    fwd = O.layer(*(inp[x] for x in "qkvg"), p, k, kept=sel, kept_ref=sel_ref)
    bwd = O.layer_backward(d_out, fwd, p)

    # combine backward, on the GPU's own o_fine (bf16) so that only this step is measured
    d_out_t = f64(layer.d_out_t)
    assert np.array_equal(d_out_t, bwd["d_out_t"])
    o_fine_gpu = f64(layer.o_fine_t)
    want_delta = (d_out_t * o_fine_gpu).sum(axis=-1)
    assert_rel(f64(layer.delta), want_delta, 1e-4, 1e-4, "delta")
    _, dg_t, doc = O.gate_combine_backward(d_out_t, o_fine_gpu, f64(layer.g_t), f64(layer.o_coarse), p)
    assert_rel(f64(layer.dg_t), dg_t, 2 ** -8, 2 ** -8, "d_gate_t")
    assert_rel(f64(layer.d_o_coarse), doc, 1e-4, 1e-4, "d_o_coarse")

    # coarse backward, on the GPU's pooled means and d_o_coarse
    qbar, kbar, vbar = (f64(t) for t in vsa.pooled_slots(plan, layer.ws, w.B, w.H, w.D))
    want = O.coarse_attention_backward(qbar, kbar, vbar, w.D ** -0.5, f64(layer.d_o_coarse))
    for got, ref, name in zip(layer.d_bar, want, ("d_qbar", "d_kbar", "d_vbar")):
        assert_rel(f64(got), ref, 1e-3, 1e-3, name)

    # the whole backward, natural order, against the oracle end to end
    for got, name in zip(grads, ("dq", "dk", "dv", "dg")):
        assert_rel(f64(got), bwd[name], what=name)
    # the forward it rests on
    assert_rel(f64(out), fwd["out"], what="out")


@pytest.mark.parametrize("w,k_ref", [CASES[0], CASES[2], CASES[8]],
                         ids=lambda c: getattr(c, "name", str(c)))
def test_sparse_attn_backward_without_pooling_term(w, k_ref):
    """vsa_sparse_attn_backward with no pooled gradients: the fine-attention
    gradients alone, against the oracle's fine backward."""
    inp, d_out, plan, k, layer, _, _ = _run(w, k_ref)
    dq, dk, dv = vsa.vsa_sparse_attn_backward(
        plan, layer.q_t, layer.k_t, layer.v_t, layer.d_out_t, layer.topk_idx, k, layer.lse,
        layer.delta, layer.bws, topk_ref=layer.topk_ref, k_ref=k_ref)
    vsa.vsa_sync_status(plan)
    p = O.plan(w.prefix, w.grid, w.tile)
    sel = layer.topk_idx.cpu().numpy().astype(np.int64)
    sel_ref = None if k_ref is None else layer.topk_ref.cpu().numpy().astype(np.int64)
    want = O.fine_backward(f64(layer.q_t), f64(layer.k_t), f64(layer.v_t), p, sel, w.D ** -0.5,
                           f64(layer.d_out_t), sel_ref)
    for got, ref, name in zip((dq, dk, dv), want, ("dq_t", "dk_t", "dv_t")):
        g = f64(got)
        assert np.all(g[..., p.row_src < 0, :] == 0.0), f"{name}: pad rows not zero"
        assert_rel(g, ref, what=name)


def test_backward_rejects_bad_arguments():
    w = TINY
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    layer = vsa.TrainingLayer(plan, 1, 2, 64, 2)
    with pytest.raises(vsa.VsaError) as e:        # workspace too small
        vsa.vsa_coarse_backward(plan, *vsa.pooled_slots(plan, layer.ws, 1, 2, 64), layer.d_o_coarse,
                                layer.bws[:16])
    assert e.value.status == 4
    with pytest.raises(vsa.VsaError) as e:        # only some pooled gradients
        vsa.vsa_sparse_attn_backward(plan, layer.q_t, layer.k_t, layer.v_t, layer.d_out_t,
                                     layer.topk_idx, 2, layer.lse, layer.delta, layer.bws,
                                     d_bar=(layer.d_bar[0], None, None))
    assert e.value.status == 1
    vsa.vsa_sync_status(plan)


def test_backward_full_size_sampled():
    """The 104,704-token, 42-head Veda layer in the benchmark's launch
    configuration (vsa.TrainingLayer): for two heads, the oracle computes the
    coarse backward of the whole head and, one tile at a time, dq of sampled
    query tiles (prefix and video), dk and dv of a sampled video key tile
    (summing over every query tile that attends to it) and d_gate of the
    sampled query tiles' rows."""
    from tile_sparse_video_b200.inputs import VEDA_104K
    w = VEDA_104K
    inp = make_inputs(w)
    d_out = make_grad_output(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    k = _keep(plan, w)
    layer = vsa.TrainingLayer(plan, w.B, w.H, w.D, k)
    layer.forward(*(inp[x].cuda() for x in "qkvg"))
    layer.backward(d_out.cuda())
    vsa.vsa_sync_status(plan)
    p = O.plan(w.prefix, w.grid, w.tile)
    R, n_p, T = p.R, p.n_prefix_tiles, p.n_tiles
    scale = w.D ** -0.5
    sel_all = layer.topk_idx.cpu().numpy().astype(np.int64)
    rng = np.random.default_rng(5)
    for h in (0, w.H - 1):
        q_t, k_t, v_t, g_t = (O.permute(inp[x][0, h].to(torch.float64).numpy(), p) for x in "qkvg")
        d_t = O.permute(d_out[0, h].to(torch.float64).numpy(), p)
        qbar, kbar, vbar = O.pool(q_t, p), O.pool(k_t, p), O.pool(v_t, p)
        _, o_coarse = O.coarse_attention(qbar, kbar, vbar, scale)
        _, dg_t, d_oc = O.gate_combine_backward(d_t, np.zeros_like(d_t), g_t, o_coarse, p)
        d_qbar, d_kbar, d_vbar = O.coarse_attention_backward(qbar, kbar, vbar, scale, d_oc)
        sel = sel_all[0, h]
        keys = lambda i: O.key_tiles(p, i, sel[i - n_p] if i >= n_p else None)
        gq, gk, gv, gg = (f64(t[0, h]) for t in (layer.dq_t, layer.dk_t, layer.dv_t, layer.dg_t))
        # dq of sampled query tiles
        for i in [0, n_p, T - 1] + list(rng.choice(np.arange(n_p, T), 2, replace=False)):
            n = p.block_len[i]
            rows = slice(i * R, i * R + n)
            _, dq, _, _ = O.fine_tile_backward(q_t, k_t, v_t, p, i, keys(i), scale, d_t[rows])
            assert_rel(gq[rows], dq + d_qbar[i] / n, what=f"dq h{h} tile {i}")
            assert_rel(gg[rows], dg_t[rows], 2 ** -8, 2 ** -8, f"d_gate h{h} tile {i}")
        # dk, dv of a sampled video key tile (a prefix key tile is attended by all
        # 818 query tiles, too many for the oracle here; the small layouts cover it)
        for j in [int(rng.integers(n_p, T))]:
            n = p.block_len[j]
            dk = np.zeros((n, w.D))
            dv = np.zeros((n, w.D))
            for i in range(T):
                ks = keys(i)
                if j not in ks:
                    continue
                rows_i = slice(i * R, i * R + p.block_len[i])
                key_rows, _, dki, dvi = O.fine_tile_backward(q_t, k_t, v_t, p, i, ks, scale, d_t[rows_i])
                at = np.searchsorted(key_rows, j * R)
                dk += dki[at: at + n]
                dv += dvi[at: at + n]
            rows = slice(j * R, j * R + n)
            assert_rel(gk[rows], dk + d_kbar[j] / n, what=f"dk h{h} tile {j}")
            assert_rel(gv[rows], dv + d_vbar[j] / n, what=f"dv h{h} tile {j}")
