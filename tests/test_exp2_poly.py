"""Pins the FMA-pipe exp2 of the attention kernel against the mathematics.

The kernel computes 2^x as 2^n * p(f), with n = round(x) and
f = x - n in [-1/2, 1/2]. This test reads the coefficients of p from the
kernel header and checks, in fp64:
  - the relative error of p against 2^f on a dense grid;
  - p(0) = 1;
  - continuity where n switches, p(1/2) = 2 p(-1/2).
It then replays the range reduction with float32 rounding in numpy, over
the input range the softmax uses ([-125, 8]), against numpy's exp2.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "block_sparse_masked_tile_b200", "csrc", "attn_fwd.cuh")


def coefficients():
    text = open(HEADER).read()
    c = {}
    for k in ("C1", "C2", "C3"):
        m = re.search(rf"constexpr float kExp2{k} = ([0-9.eE+-]+)f;", text)
        assert m, k
        c[k] = float(np.float32(float(m.group(1))))
    return 1.0, c["C1"], c["C2"], c["C3"]


def poly(f, c):
    return ((c[3] * f + c[2]) * f + c[1]) * f + c[0]


def test_polynomial_error_bound():
    c = coefficients()
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(poly(f, c) - np.exp2(f)) / np.exp2(f)
    assert rel.max() < 1.1e-4
    assert poly(0.0, c) == 1.0
    assert abs(poly(0.5, c) - 2 * poly(-0.5, c)) < 1e-6


def test_range_reduction_in_float32():
    c = [np.float32(v) for v in coefficients()]
    x = np.linspace(-125.0, 8.0, 400001).astype(np.float32)
    rnd = np.float32(12582912.0)
    t = (x + rnd).astype(np.float32)
    n = (t - rnd).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = (((c[3] * f + c[2]) * f + c[1]) * f + c[0]).astype(np.float32)
    bits = q.view(np.int32) + (t.view(np.int32) << 23)
    y = bits.view(np.float32).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(y - want) / want
    assert rel.max() < 2e-4
    assert np.all(np.abs(f) <= 0.5)
