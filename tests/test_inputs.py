"""The seeded input generator: deterministic, and a head/batch subset is
bit-identical to the same slice of the full draw."""
import torch

from tile_sparse_video_b200.inputs import TINY, SMALL, make_inputs, sweep_workloads


def test_inputs_deterministic_and_sliceable():
    a = make_inputs(TINY)
    b = make_inputs(TINY)
    for k in "qkvg":
        assert a[k].dtype == torch.bfloat16
        assert a[k].shape == (1, 2, TINY.n_tokens, 64)
        assert torch.equal(a[k], b[k])
    c = make_inputs(TINY, heads=[1])
    for k in "qkvg":
        assert torch.equal(c[k][:, 0], a[k][:, 1])


def test_sweep_workloads_shapes():
    ws = sweep_workloads()
    assert len(ws) == 40
    assert all(w.B == 2 for w in ws)
    assert {w.grid[0] for w in ws} == {16, 32, 64, 102, 104}
