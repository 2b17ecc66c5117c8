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


def test_grad_output_deterministic_sliceable_and_independent():
    """The backward's upstream gradient: seeded, bf16 [B,H,N,D], a head subset
    equals the same slice of the full draw, and it is not a copy of any forward
    input (its own generator)."""
    from dataclasses import replace
    from tile_sparse_video_b200.inputs import make_grad_output
    w = replace(TINY, B=2)
    a = make_grad_output(w)
    assert a.dtype == torch.bfloat16 and a.shape == (2, 2, w.n_tokens, 64)
    assert torch.equal(a, make_grad_output(w))
    assert torch.equal(make_grad_output(w, batch=[1], heads=[1])[0, 0], a[1, 1])
    inp = make_inputs(w)
    for k in "qkvg":
        assert not torch.equal(a, inp[k])
    assert not torch.equal(a[0], a[1])
