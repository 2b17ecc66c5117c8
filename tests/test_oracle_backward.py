"""Pins for the oracle's backward pass, computed without its own code paths.

* central finite differences of the forward oracle (the selection held fixed,
  since it passes no gradient): the directional derivative of
  L = sum(d_out * out) along random directions of q, k, v and g, and along
  single coordinates (prefix, video and ragged-tile tokens);
* the dense special case: with every video tile kept and the gate at -inf the
  layer is plain softmax attention over all tokens, whose gradients come from
  torch autograd on the library attention routine in fp64;
* adjoint identities of the pooling and permutation steps.
The last test plants mistakes in the backward and checks that a pin catches
each one.
"""
import numpy as np
import pytest
import torch

import oracle as O


def _inputs(prefix, grid, tile, B, H, D, seed, scale_v=1.0):
    p = O.plan(prefix, grid, tile)
    rng = np.random.default_rng(seed)
    q, k, v, g, d_out = (rng.standard_normal((B, H, p.n_tokens, D)) for _ in range(5))
    return p, q, k, v * scale_v, g, d_out


def _loss(q, k, v, g, p, kk, kept, kept_ref, d_out):
    f = O.layer(q, k, v, g, p, kk, kept=kept, kept_ref=kept_ref)
    return float((f["out"] * d_out).sum())


CASES = [
    # prefix, grid, tile, B, H, D, k, k_ref
    ((40, 70), (4, 8, 8), (4, 4, 4), 1, 2, 16, 2, None),
    ((5, 0, 64, 65), (5, 6, 7), (4, 4, 4), 2, 1, 8, 3, None),   # empty segment, ragged cubes
    ((40, 70), (4, 8, 8), (4, 4, 4), 1, 1, 16, 2, 1),           # reference thinning
    ((256, 3), (4, 17, 9), (4, 8, 4), 1, 1, 8, 2, None),        # 128-row tiles
]


@pytest.mark.parametrize("case", CASES, ids=["tiny", "ragged_b2", "ref_thin", "r128"])
def test_backward_matches_finite_differences(case):
    prefix, grid, tile, B, H, D, kk, k_ref = case
    p, q, k, v, g, d_out = _inputs(prefix, grid, tile, B, H, D, seed=len(prefix) + D)
    fwd = O.layer(q, k, v, g, p, kk, k_ref=k_ref)
    bwd = O.layer_backward(d_out, fwd, p)
    kept, kept_ref = fwd["topk"], fwd["topk_ref"]
    rng = np.random.default_rng(7)
    eps = 1e-5
    args = dict(q=q, k=k, v=v, g=g)
    for name in ("q", "k", "v", "g"):
        u = rng.standard_normal(args[name].shape)
        plus = dict(args, **{name: args[name] + eps * u})
        minus = dict(args, **{name: args[name] - eps * u})
        fd = (_loss(**plus, p=p, kk=kk, kept=kept, kept_ref=kept_ref, d_out=d_out)
              - _loss(**minus, p=p, kk=kk, kept=kept, kept_ref=kept_ref, d_out=d_out)) / (2 * eps)
        an = float((bwd["d" + name] * u).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)
    # single coordinates: first prefix token, last token, a token of a ragged tile
    tokens = [0, p.n_tokens - 1, int(p.row_src[p.R * (p.n_tiles - 1)])]
    for name in ("q", "k", "v", "g"):
        for n in tokens:
            for d in (0, D - 1):
                u = np.zeros(args[name].shape)
                u[0, 0, n, d] = 1.0
                plus = dict(args, **{name: args[name] + eps * u})
                minus = dict(args, **{name: args[name] - eps * u})
                fd = (_loss(**plus, p=p, kk=kk, kept=kept, kept_ref=kept_ref, d_out=d_out)
                      - _loss(**minus, p=p, kk=kk, kept=kept, kept_ref=kept_ref, d_out=d_out)) / (2 * eps)
                an = bwd["d" + name][0, 0, n, d]
                assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, n, d, fd, an)


@pytest.mark.parametrize("prefix,grid,tile", [((40, 70), (4, 8, 8), (4, 4, 4)),
                                              ((256, 3), (4, 17, 9), (4, 8, 4))])
def test_backward_dense_case_is_library_attention_gradient(prefix, grid, tile):
    """k = n_v and a gate of -inf: out = softmax attention over all tokens."""
    B, H, D = 1, 2, 16
    p, q, k, v, _, d_out = _inputs(prefix, grid, tile, B, H, D, seed=3)
    g = np.full(q.shape, -np.inf)
    fwd = O.layer(q, k, v, g, p, p.n_video_tiles)
    bwd = O.layer_backward(d_out, fwd, p)
    t = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v)]
    out = torch.nn.functional.scaled_dot_product_attention(*t, scale=D ** -0.5)
    out.backward(torch.from_numpy(d_out))
    for name, ref in zip(("dq", "dk", "dv"), t):
        np.testing.assert_allclose(bwd[name], ref.grad.numpy(), rtol=0, atol=1e-12)
    assert np.all(bwd["dg"] == 0.0)


def test_pool_and_permute_adjoints():
    """<pool(x), y> = <x, pool_backward(y)> and <permute(x), y> = <x, unpermute(y)>."""
    p = O.plan((5, 0, 64, 65), (5, 6, 7), (4, 4, 4))
    rng = np.random.default_rng(11)
    x_t = rng.standard_normal((2, p.n_padded, 3))
    x_t[:, p.row_src < 0] = 0.0
    y = rng.standard_normal((2, p.n_tiles, 3))
    assert np.isclose((O.pool(x_t, p) * y).sum(), (x_t * O.pool_backward(y, p)).sum(), rtol=1e-13)
    x = rng.standard_normal((2, p.n_tokens, 3))
    z = rng.standard_normal((2, p.n_padded, 3))
    assert np.isclose((O.permute(x, p) * z).sum(), (x * O.unpermute(z, p)).sum(), rtol=1e-13)
    assert np.all(O.pool_backward(y, p)[:, p.row_src < 0] == 0.0)


def test_backward_closed_forms():
    """One tile per query, constant d_out on a T = 1 layout: the coarse output
    is the pooled v, so d_vbar = d_o_coarse and the pooled q, k get nothing."""
    qbar = np.random.default_rng(1).standard_normal((1, 4))
    kbar = np.random.default_rng(2).standard_normal((1, 4))
    vbar = np.random.default_rng(3).standard_normal((1, 4))
    d = np.random.default_rng(4).standard_normal((1, 4))
    dq, dk, dv = O.coarse_attention_backward(qbar, kbar, vbar, 0.5, d)
    assert np.allclose(dq, 0.0, atol=1e-15) and np.allclose(dk, 0.0, atol=1e-15)
    assert np.allclose(dv, d, rtol=1e-15)
    # gate at 0: d_g = d_out * o_coarse / 4, d_o_coarse = sum of d_out / 2
    p = O.plan((), (4, 4, 4), (4, 4, 4))
    o_c = np.random.default_rng(5).standard_normal((1, 4))
    d_out_t = np.random.default_rng(6).standard_normal((64, 4))
    d_f, d_g, d_oc = O.gate_combine_backward(d_out_t, np.zeros((64, 4)), np.zeros((64, 4)), o_c, p)
    assert np.allclose(d_g, d_out_t * o_c / 4, rtol=1e-15)
    assert np.allclose(d_oc, d_out_t.sum(axis=0, keepdims=True) / 2, rtol=1e-14)
    assert np.array_equal(d_f, d_out_t)


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_planted_backward_mistakes_are_caught(monkeypatch):
    import oracle.vsa_oracle as V
    fd = lambda: test_backward_matches_finite_differences(CASES[0])

    # 1. softmax backward without the row-sum term
    monkeypatch.setattr(V, "softmax_backward", lambda prob, d: prob * d)
    assert _fails(fd)
    monkeypatch.undo()

    # 2. pooling backward that does not divide by the live-row count
    def undivided(d_bar, p):
        out = np.zeros(d_bar.shape[:-2] + (p.n_padded, d_bar.shape[-1]))
        for t in range(p.n_tiles):
            out[..., t * p.R: t * p.R + p.block_len[t], :] = d_bar[..., t: t + 1, :]
        return out
    monkeypatch.setattr(V, "pool_backward", undivided)
    assert _fails(fd)
    monkeypatch.undo()

    # 3. gate gradient through sigmoid instead of its derivative
    orig = V.gate_combine_backward
    def wrong_gate(d_out_t, o_fine, g_t, o_coarse, p):
        d_f, _, d_oc = orig(d_out_t, o_fine, g_t, o_coarse, p)
        tile_of_row = np.repeat(np.arange(p.n_tiles), p.R)
        d = d_f
        return d_f, d * o_coarse[..., tile_of_row, :] * V.sigmoid(g_t), d_oc
    monkeypatch.setattr(V, "gate_combine_backward", wrong_gate)
    assert _fails(fd)
    monkeypatch.undo()

    # 4. key gradient without the softmax scale
    orig_tile = V.fine_tile_backward
    def unscaled_dk(q_t, k_t, v_t, p, i, tiles, scale, d_o):
        rows, dq, dk, dv = orig_tile(q_t, k_t, v_t, p, i, tiles, scale, d_o)
        return rows, dq, dk / scale, dv
    monkeypatch.setattr(V, "fine_tile_backward", unscaled_dk)
    assert _fails(fd)
    monkeypatch.undo()

    # 5. coarse key gradient from the untransposed score gradient
    orig_c = V.coarse_attention_backward
    def untransposed(qbar, kbar, vbar, scale, d_o):
        dq, dk, dv = orig_c(qbar, kbar, vbar, scale, d_o)
        s = scale * (qbar @ np.swapaxes(kbar, -1, -2))
        e = np.exp(s - s.max(axis=-1, keepdims=True))
        prob = e / e.sum(axis=-1, keepdims=True)
        d_s = V.softmax_backward(prob, d_o @ np.swapaxes(vbar, -1, -2))
        return dq, scale * (d_s @ qbar), dv
    monkeypatch.setattr(V, "coarse_attention_backward", untransposed)
    assert _fails(fd)
    monkeypatch.undo()
