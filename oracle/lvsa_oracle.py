"""fp64/integer CPU oracle: the LVSA static attention pattern (local temporal
window plus rotating equidistant global frames) as a block mask.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA product path
never imports this module, and this module imports nothing from it.

Source ("LVSA: Training-Free Sparse Attention for Long Video Diffusion",
cited as LVSA):
  [LVSA §3, attention pattern]  query frame t attends A(t) = G ∪ W(t): the
        global frames G, one every Tper frames, and a local window W(t) of up
        to 2W+1 neighbouring frames, clipped at the ends of the video.
  [LVSA §3, budget allocation]  the window bounds are expanded to make up for
        clipping and for overlap with G, so that every frame attends the same
        number |A(t)| = |G| + min(2W+1, T - |G|) of frames; a short loop does it.
  [LVSA §3, rotating global frames]  at denoising step s the global set is
        shifted by s modulo Tper, so every frame is global once per Tper steps.

The steps follow the page: global set, clipped window, expansion loop until the
target count, then the frame pattern is lifted to blocks of the permuted token
sequence.

Readings of points the page leaves open (each one is listed in the design notes):
  * G_s = { g in [0, T) : g = s (mod Tper) }.
  * expansion: each pass adds exactly the current deficit (target - |A|) to
    the window, the larger half after t and the smaller half before t; a side
    that reaches the end of the video gives the rest to the other side. A pass
    can never overshoot (each added frame raises |A| by at most one), and it
    repeats while added frames fall on global frames.
  * blocks: key block j is attended by query block i when some valid token of
    i lies in a frame tq and some valid token of j in a frame of A(tq).
"""

from __future__ import annotations

import numpy as np

from .fvattn_oracle import num_blocks


def global_frames(T: int, Tper: int, step: int) -> set:
    """G_s: every Tper-th frame, starting at step mod Tper."""
    r = step % Tper
    return set(range(r, T, Tper))


def target_count(T: int, W: int, Tper: int, step: int) -> int:
    g = len(global_frames(T, Tper, step))
    return g + min(2 * W + 1, T - g)


def attended_frames(t: int, T: int, W: int, Tper: int, step: int) -> tuple[set, int, int]:
    """A(t) and the final window bounds [lo, hi] for query frame t."""
    G = global_frames(T, Tper, step)
    target = target_count(T, W, Tper, step)
    lo, hi = max(0, t - W), min(T - 1, t + W)
    while True:
        A = G | set(range(lo, hi + 1))
        deficit = target - len(A)
        if deficit <= 0:
            return A, lo, hi
        right = min(T - 1 - hi, (deficit + 1) // 2)
        left = min(lo, deficit - right)
        right = min(T - 1 - hi, deficit - left)
        if left == 0 and right == 0:      # cannot grow (does not happen: target <= T)
            return A, lo, hi
        lo -= left
        hi += right


def frame_mask(T: int, W: int, Tper: int, step: int) -> np.ndarray:
    """[T, T] bool: entry (tq, tk) true when query frame tq attends key frame tk."""
    m = np.zeros((T, T), dtype=bool)
    for t in range(T):
        A, _, _ = attended_frames(t, T, W, Tper, step)
        m[t, sorted(A)] = True
    return m


def block_frames(perm: np.ndarray, T: int, Hh: int, W_: int, N: int, bs: int) -> list:
    """Frames of the valid tokens of each block of the permuted sequence."""
    nb = num_blocks(N, bs)
    frames = []
    for i in range(nb):
        src = np.asarray(perm[i * bs:min((i + 1) * bs, N)])
        frames.append(set(int(v) for v in np.unique(src // (Hh * W_))))
    return frames


def lvsa_block_mask(perm: np.ndarray, grid, bs: int, W: int, Tper: int, step: int) -> np.ndarray:
    """[nb, nb] bool block mask of the LVSA pattern for a token order ``perm``.

    ``grid`` = (T, Hh, Wd): the latent video extents; ``perm[pos]`` is the
    raster index of the token at position ``pos`` of the permuted sequence.
    """
    T, Hh, Wd = grid
    N = T * Hh * Wd
    fm = frame_mask(T, W, Tper, step)
    bf = block_frames(perm, T, Hh, Wd, N, bs)
    nb = len(bf)
    out = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        allowed = set()
        for tq in bf[i]:
            allowed |= set(np.nonzero(fm[tq])[0].tolist())
        for j in range(nb):
            out[i, j] = bool(bf[j] & allowed)
    return out
