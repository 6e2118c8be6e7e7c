"""Pins of the Hilbert-order oracle (no GPU).

  * hand-derived curves in tests/golden/hilbert_orders.txt: the textbook 2-D
    order-2 curve (either orientation) and the 3-D order-1 curve (the reflected
    Gray code);
  * defining properties on cubes of side 2^b: a bijection onto [0, 2^(nb)),
    consecutive points one unit step apart (continuity), every aligned sub-cube
    of side 2^k visited in one contiguous run (locality at every scale), and
    starting at the origin;
  * the grid order written a second way: the full cube's curve enumerated
    point by point, filtered to the grid;
  * planted mistakes (no Gray step, Morton order, raster order) fail a pin.
"""

import itertools
import os

import numpy as np
import pytest

from oracle import hilbert_oracle as Hb

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hilbert_orders.txt")


def _golden(tag, n):
    for line in open(GOLDEN):
        if line.startswith(tag + ":"):
            v = [int(t) for t in line.split(":")[1].split()]
            return [tuple(v[i:i + n]) for i in range(0, len(v), n)]
    raise KeyError(tag)


def _curve(n, b, index_fn=None):
    """Cube points sorted by index (the curve), as a list of coordinate tuples."""
    f = index_fn or (lambda c: Hb.hilbert_index(c, b))
    pts = list(itertools.product(range(1 << b), repeat=n))
    return sorted(pts, key=f)


def test_2d_order2_is_the_textbook_curve():
    want = _golden("2d4", 2)
    got = _curve(2, 2)
    assert got == want or got == [(y, x) for (x, y) in want]


def test_3d_order1_is_the_reflected_gray_code():
    assert _curve(3, 1) == _golden("3d2", 3)


def _check_hilbert_properties(pts, n, b):
    assert len(set(pts)) == len(pts) == (1 << (n * b))
    assert pts[0] == (0,) * n
    steps = np.abs(np.diff(np.array(pts), axis=0))
    assert np.all(steps.sum(axis=1) == 1), "consecutive points must be one unit step apart"
    for k in range(1, b):
        cell = [tuple(c >> k for c in p) for p in pts]
        runs = [c for i, c in enumerate(cell) if i == 0 or c != cell[i - 1]]
        assert len(runs) == len(set(runs)), f"an aligned 2^{k} sub-cube is visited twice"


@pytest.mark.parametrize("n,b", [(2, 1), (2, 3), (2, 5), (3, 1), (3, 2), (3, 3), (3, 4)])
def test_curve_properties_on_cubes(n, b):
    _check_hilbert_properties(_curve(n, b), n, b)


@pytest.mark.parametrize("T,Hh,W", [(3, 5, 7), (2, 8, 8), (5, 3, 9), (1, 6, 10), (4, 4, 4), (7, 1, 1)])
def test_grid_order_is_the_cube_curve_restricted_to_the_grid(T, Hh, W):
    b = Hb.bits_for(max(T, Hh, W))
    full = _curve(3, b)
    want = [(t * Hh + y) * W + x for (t, y, x) in full if t < T and y < Hh and x < W]
    got = Hb.hilbert_order(T, Hh, W)
    assert np.array_equal(got, want)
    assert sorted(got.tolist()) == list(range(T * Hh * W))


def test_bits_for():
    assert [Hb.bits_for(e) for e in (1, 2, 3, 4, 5, 8, 9, 80)] == [1, 1, 2, 2, 3, 3, 4, 7]


# ---------------------------------------------------------------- planted mistakes

def _no_gray(coords, b):
    X = [int(c) for c in coords]
    return Hb.transpose_to_index(X, b)          # skips the transform: Morton (Z) order


def _raster(coords, b):
    h = 0
    for c in coords:
        h = (h << b) | int(c)
    return h


def _skip_low_gray(coords, b):
    # the inverse-undo loop without the final Gray encode
    X = [int(c) for c in coords]
    n = len(X)
    Q = 1 << (b - 1)
    while Q > 1:
        P = Q - 1
        for i in range(n):
            if X[i] & Q:
                X[0] ^= P
            else:
                t = (X[0] ^ X[i]) & P
                X[0] ^= t
                X[i] ^= t
        Q >>= 1
    return Hb.transpose_to_index(X, b)


@pytest.mark.parametrize("bad", [_no_gray, _raster, _skip_low_gray])
def test_planted_order_mistakes_are_caught(bad):
    with pytest.raises(AssertionError):
        _check_hilbert_properties(_curve(3, 3, lambda c: bad(c, 3)), 3, 3)
