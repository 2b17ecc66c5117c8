"""The FMA-pipe exp2 of the attention kernel, checked against its error bound.

The attention kernel has an optional FMA-pipe exp2 (off by default: the
VSA_EXP2_FMA_SHARE build knob selects which share of the exponentials it
takes off the MUFU unit), a Cody-Waite + degree-3 polynomial of its own.  This
test reads the coefficients
from the kernel source, replays the same float32 operations in numpy and
checks the relative error against 2^x over the whole range the softmax feeds
it (x in [-125, 8]: scores minus a running max, which may lag by up to 8)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "tile_sparse_video_b200", "csrc", "sparse_attn.cu")


def coefficients():
    text = open(SRC).read()
    c = {int(m.group(1)): np.float32(float(m.group(2)))
         for m in re.finditer(r"constexpr float kExp2C(\d) = ([-0-9.eE+]+)f;", text)}
    assert sorted(c) == [0, 1, 2, 3]
    return c


def exp2_fma(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
    p = (c[3] * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    return (p.view(np.int32) + (t.view(np.int32) << 23)).astype(np.int32).view(np.float32)


def test_exp2_fma_relative_error_bound():
    c = coefficients()
    x = np.concatenate([np.linspace(-125, 8, 1_000_001), np.arange(-125, 9).astype(np.float64),
                        np.arange(-125, 8) + 0.5]).astype(np.float32)
    got = exp2_fma(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 3e-4, rel.max()            # bf16 rounding alone is up to 2^-9 ~ 2e-3


def test_exp2_fma_limits():
    c = coefficients()
    y = exp2_fma(np.array([-np.inf, -1e30, -126.0, 0.0], dtype=np.float32), c)
    assert np.all(y[:3] <= 2.0 ** -124) and np.all(y[:3] > 0)    # masked scores: ~0
    assert abs(float(y[3]) - 1.0) < 1e-4
