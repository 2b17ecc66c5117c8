"""GPU parity of the head projection (vsa_project, a tcgen05 GEMM) against the
fp64 oracle on the same bf16 inputs.

Every output is one bf16 rounding (relative 2^-9) of an fp32 sum of C
products; the bound checked is 2^-8 relative to the largest |y| of the
output row plus 1e-6 absolute (fp32 accumulation over C <= 5376 terms
contributes ~1e-6 relative).  Shapes cover a partial last M tile, H*D not a
multiple of the 256-column N tile, C not a multiple of the 64-wide K block,
D = 64 and 128, both activations, and B = 2 (rows of two batch elements in
one M tile)."""
import numpy as np
import pytest
import torch

import oracle as O
from tile_sparse_video_b200 import vsa
from tile_sparse_video_b200.inputs import SMALL, TINY, VEDA_104K, Workload, make_projection_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda(libvsa):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _check(got, want):
    got = got.to(torch.float64).cpu().numpy()
    assert np.all(np.isfinite(got))
    scale = np.abs(want).max(axis=-1, keepdims=True)
    err = np.abs(got - want)
    bound = 2.0 ** -8 * scale + 1e-6
    assert np.all(err <= bound), float((err / (scale + 1e-30)).max())


def _case(name, prefix, grid, tile, B, H, D, C, seed):
    return Workload(name, B=B, H=H, D=D, prefix=prefix, grid=grid, tile=tile, keep_tiles=1,
                    gate_width=C, gate_std=0.05, seed_base=seed)


CASES = [
    (_case("tiny_gate", TINY.prefix, TINY.grid, TINY.tile, 1, 2, 128, 64, 11), False),
    (_case("d64_hd192_c200_b2", (40, 70), (4, 8, 8), (4, 4, 4), 2, 3, 64, 200, 12), True),
    (_case("hd384_c520", (100,), (8, 16, 8), (4, 8, 4), 1, 3, 128, 520, 13), False),
    (SMALL, True),
]


@pytest.mark.parametrize("w,sig", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_projection_parity(w, sig):
    inp = make_projection_inputs(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    y = vsa.vsa_project(plan, inp["x"].cuda(), inp["w"].cuda(), w.H, w.D, sigmoid=sig)
    vsa.vsa_sync_status(plan)
    want = O.project(inp["x"], inp["w"], w.H, w.D, act="sigmoid" if sig else None)
    _check(y, want)


@pytest.mark.parametrize("H", [42, 56], ids=["h42", "h56"])
def test_projection_full_size_sampled(H):
    """The gate projection at the 104,704-token Veda size (C = 5,376 ->
    42 x 128, and the 56-head layout with inner width 7,168): every output of
    98 sampled rows against fp64."""
    from dataclasses import replace
    w = VEDA_104K if H == VEDA_104K.H else replace(VEDA_104K, name=f"veda_h{H}", H=H)
    inp = make_projection_inputs(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    y = vsa.vsa_project(plan, inp["x"].cuda(), inp["w"].cuda(), w.H, w.D)
    vsa.vsa_sync_status(plan)
    rows = np.sort(np.random.default_rng(3).choice(plan.n_tokens, 96, replace=False))
    rows = np.unique(np.concatenate([rows, [0, plan.n_tokens - 1]]))
    want = O.project(inp["x"][:, rows], inp["w"], w.H, w.D)
    _check(y[:, :, rows], want)


def test_projection_rejects_bad_arguments():
    w = TINY
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    x = torch.zeros(1, plan.n_tokens, 60, dtype=torch.bfloat16, device="cuda")
    wt = torch.zeros(256, 60, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vsa.VsaError) as e:           # C not a multiple of 8
        vsa.vsa_project(plan, x, wt, 2, 128)
    assert e.value.status == 1
    vsa.vsa_sync_status(plan)


# --------------------------------------------------------------------------
# Tile before projecting: vsa_permute_rows + vsa_project_tiled
# --------------------------------------------------------------------------

TILED_CASES = [
    _case("tiled_tiny", TINY.prefix, TINY.grid, TINY.tile, 1, 2, 128, 64, 21),
    _case("tiled_ragged_b2", (5, 0, 64, 65), (5, 6, 7), (4, 4, 4), 2, 3, 64, 200, 22),
    _case("tiled_r128", (256, 3), (8, 17, 9), (4, 8, 4), 1, 3, 128, 520, 23),
]


@pytest.mark.parametrize("w", TILED_CASES, ids=lambda c: c.name)
def test_permute_rows_bit_exact(w):
    """x_t[b, untile[n]] = x[b, n], pad rows zero, for rows of any width."""
    inp = make_projection_inputs(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    x_t = vsa.vsa_permute_rows(plan, inp["x"].cuda())
    vsa.vsa_sync_status(plan)
    p = O.plan(w.prefix, w.grid, w.tile)
    assert np.array_equal(x_t.cpu().to(torch.float64).numpy(), O.permute(inp["x"].to(torch.float64).numpy(), p))


@pytest.mark.parametrize("w,sig", [(TILED_CASES[0], False), (TILED_CASES[1], True), (TILED_CASES[2], False)],
                         ids=lambda c: getattr(c, "name", str(c)))
def test_project_tiled_equals_project_then_permute(w, sig):
    """Projecting the tiled input gives the tiled projection: bit-identical to
    vsa_permute(vsa_project(x)) on live rows (the same row products in the same
    order), act(0) on pad rows, and within the projection bound of the oracle."""
    inp = make_projection_inputs(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    x, wt = inp["x"].cuda(), inp["w"].cuda()
    y_t = vsa.vsa_project_tiled(plan, vsa.vsa_permute_rows(plan, x), wt, w.H, w.D, sigmoid=sig)
    ref = vsa.vsa_permute(plan, vsa.vsa_project(plan, x, wt, w.H, w.D, sigmoid=sig))
    vsa.vsa_sync_status(plan)
    p = O.plan(w.prefix, w.grid, w.tile)
    live = torch.from_numpy(p.row_src >= 0).cuda()
    assert torch.equal(y_t[:, :, live], ref[:, :, live])
    pad = y_t[:, :, ~live].to(torch.float32)
    assert torch.all(pad == (0.5 if sig else 0.0))
    want = O.permute(O.project(inp["x"], inp["w"], w.H, w.D, act="sigmoid" if sig else None), p)
    got = y_t.cpu().to(torch.float64).numpy()[:, :, p.row_src >= 0]
    _check(torch.from_numpy(got), want[:, :, p.row_src >= 0])


def test_tiled_input_projection_full_size():
    """The Veda layer input (104,704 tokens x 5,376) through
    vsa.TiledInputProjection: q_t equals vsa_permute(vsa_project(x, w_q))
    element for element."""
    w = VEDA_104K
    inp = make_projection_inputs(w)
    plan = vsa.Plan(w.prefix, w.grid, w.tile)
    x, wt = inp["x"].cuda(), inp["w"].cuda()
    proj = vsa.TiledInputProjection(plan, w.B, w.H, w.D, w.gate_width)
    q_t, k_t, v_t, g_t = proj(x, wt, wt, wt, wt)
    ref = vsa.vsa_permute(plan, vsa.vsa_project(plan, x, wt, w.H, w.D))
    vsa.vsa_sync_status(plan)
    assert torch.equal(q_t, ref) and torch.equal(g_t, ref)
