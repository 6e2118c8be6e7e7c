"""Integer CPU oracle: Hilbert-curve token order for the latent video grid.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA product path
never imports this module, and this module imports nothing from it.

Sources:
  [FVAttn §3.1]  blocks are reordered along a Hilbert curve so that tokens that
                 are neighbours in space fall into nearby blocks at every scale.
  [GSRS §A.6]    a generalized Hilbert curve groups nearby spatio-temporal
                 tokens into compact blocks; it is applied in every experiment.
  J. Skilling, "Programming the Hilbert curve", AIP Conf. Proc. 707, 381 (2004):
                 the n-dimensional Hilbert index through the "transpose" form
                 (an in-place transform of the coordinates whose bits,
                 interleaved, are the index).

Readings of points the pages leave open (each one is listed in the design notes):
  * the curve is 3-D over (t, y, x), on the smallest cube of side 2^b that holds
    the grid (b = bits of the largest extent), and tokens are ordered by their
    index on it; the grid is a sub-box of the cube, so this "generalizes" the
    curve to any extents by restriction (the order is continuous on cubes and
    keeps every aligned sub-cube contiguous);
  * axis order: t is the first coordinate, then y, then x;
  * as for tiles, the ordered sequence is cut into blocks of bs tokens and
    padded at the tail only.
"""

from __future__ import annotations

import numpy as np


def bits_for(extent: int) -> int:
    """Bits b such that 2^b >= extent (at least 1)."""
    b = 1
    while (1 << b) < extent:
        b += 1
    return b


def axes_to_transpose(coords, b: int) -> list:
    """Skilling's forward transform: coordinates (b bits each) -> transposed index."""
    X = [int(c) for c in coords]
    n = len(X)
    M = 1 << (b - 1)
    # Undo the excess work of the recursion, from the top bit down.
    Q = M
    while Q > 1:
        P = Q - 1
        for i in range(n):
            if X[i] & Q:
                X[0] ^= P                          # invert the low bits of axis 0
            else:
                t = (X[0] ^ X[i]) & P              # exchange low bits of axes 0 and i
                X[0] ^= t
                X[i] ^= t
        Q >>= 1
    # Gray encode.
    for i in range(1, n):
        X[i] ^= X[i - 1]
    t = 0
    Q = M
    while Q > 1:
        if X[n - 1] & Q:
            t ^= Q - 1
        Q >>= 1
    for i in range(n):
        X[i] ^= t
    return X


def transpose_to_index(X, b: int) -> int:
    """Interleave the transposed form: the top bit of axis 0 is the index's top bit."""
    n = len(X)
    h = 0
    for q in range(b - 1, -1, -1):
        for i in range(n):
            h = (h << 1) | ((X[i] >> q) & 1)
    return h


def hilbert_index(coords, b: int) -> int:
    return transpose_to_index(axes_to_transpose(coords, b), b)


def hilbert_order(T: int, Hh: int, W: int) -> np.ndarray:
    """perm[pos] = raster index (t*Hh + y)*W + x of the pos-th token along the curve."""
    b = bits_for(max(T, Hh, W))
    keys = np.empty(T * Hh * W, dtype=np.int64)
    for t in range(T):
        for y in range(Hh):
            for x in range(W):
                keys[(t * Hh + y) * W + x] = hilbert_index((t, y, x), b)
    return np.argsort(keys, kind="stable")
