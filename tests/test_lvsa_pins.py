"""Pins of the LVSA mask oracle (no GPU).

Each check ties the oracle to something other than itself:
  * hand-derived attended sets in tests/golden/lvsa_frames.txt;
  * the page's own claims: every frame attends the same number
    |G| + min(2W+1, T-|G|) of frames; the global frames and the clipped local
    window are always attended; rotating over Tper steps makes every frame
    global once [LVSA §3];
  * special cases: Tper = 1 or a window covering the video give dense attention;
  * the block mask written a second way: a token-level mask from the frame
    pattern, pooled with "any" over each block pair (NumPy indexing);
  * frame-aligned blocks reproduce the frame pattern exactly;
  * planted mistakes in copies of the oracle's steps.
"""

import os

import numpy as np
import pytest

import oracle as O
from oracle import lvsa_oracle as L

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "lvsa_frames.txt")


def _golden():
    cases = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, tail = line.split(":")
        cases.append((tuple(int(v) for v in head.split()), [int(v) for v in tail.split()]))
    return cases


@pytest.mark.parametrize("case", _golden(), ids=lambda c: "T%d-W%d-P%d-s%d-t%d" % c[0])
def test_golden_attended_frames(case):
    (T, W, Tper, s, t), want = case
    A, _, _ = L.attended_frames(t, T, W, Tper, s)
    assert sorted(A) == want


def _sweep():
    for T in (1, 2, 3, 5, 8, 13, 21, 30):
        for W in (0, 1, 2, 3, 6):
            for Tper in (1, 2, 3, 5, 8):
                for s in (0, 1, Tper + 2):
                    yield T, W, Tper, s


def test_uniform_count_and_containment_over_a_sweep():
    for T, W, Tper, s in _sweep():
        G = L.global_frames(T, Tper, s)
        target = len(G) + min(2 * W + 1, T - len(G))
        assert L.target_count(T, W, Tper, s) == target
        for t in range(T):
            A, lo, hi = L.attended_frames(t, T, W, Tper, s)
            assert len(A) == target, (T, W, Tper, s, t)
            assert G <= A
            assert set(range(max(0, t - W), min(T, t + W + 1))) <= A
            assert lo <= t <= hi and A == G | set(range(lo, hi + 1))


def test_global_frames_are_equidistant_and_rotate_through_every_frame():
    T, Tper = 21, 5
    for s in range(12):
        G = sorted(L.global_frames(T, Tper, s))
        assert G[0] == s % Tper and np.all(np.diff(G) == Tper)
    seen = {}
    for s in range(Tper):
        for g in L.global_frames(T, Tper, s):
            seen[g] = seen.get(g, 0) + 1
    assert sorted(seen) == list(range(T)) and set(seen.values()) == {1}


@pytest.mark.parametrize("T,W,Tper", [(9, 1, 1), (9, 8, 4), (9, 20, 3), (1, 0, 2)])
def test_dense_special_cases(T, W, Tper):
    assert L.frame_mask(T, W, Tper, 0).all()


def _token_level_block_mask(perm, grid, bs, W, Tper, s):
    T, Hh, Wd = grid
    N = T * Hh * Wd
    nb = O.num_blocks(N, bs)
    fm = L.frame_mask(T, W, Tper, s)
    frame_of_pos = np.asarray(perm)[:N] // (Hh * Wd)          # frame of each permuted position
    tok = fm[frame_of_pos[:, None], frame_of_pos[None, :]]   # [N, N] query pos x key pos
    pad = np.zeros((nb * bs, nb * bs), dtype=bool)
    pad[:N, :N] = tok
    return pad.reshape(nb, bs, nb, bs).any(axis=(1, 3))


@pytest.mark.parametrize("grid,tile,bs,W,Tper,s", [
    ((6, 4, 5), (2, 4, 4), 16, 1, 3, 0),
    ((7, 3, 6), (1, 3, 6), 16, 1, 2, 5),
    ((9, 4, 4), (2, 2, 2), 32, 2, 4, 1),
    ((5, 5, 7), (3, 2, 3), 64, 0, 2, 3),
])
def test_block_mask_equals_pooled_token_mask(grid, tile, bs, W, Tper, s):
    perm = O.tile_order(*grid, *tile)
    got = L.lvsa_block_mask(perm, grid, bs, W, Tper, s)
    want = _token_level_block_mask(perm, grid, bs, W, Tper, s)
    assert np.array_equal(got, want)
    assert got.diagonal().all()


def test_frame_aligned_blocks_reproduce_the_frame_pattern():
    # one frame of 4x4 tokens per 16-token block: block mask == frame mask
    grid = (10, 4, 4)
    perm = O.tile_order(*grid, 1, 4, 4)
    for W, Tper, s in [(1, 3, 0), (2, 4, 3), (0, 5, 7)]:
        assert np.array_equal(L.lvsa_block_mask(perm, grid, 16, W, Tper, s), L.frame_mask(10, W, Tper, s))


# ---------------------------------------------------------------- planted mistakes

def _no_expansion(t, T, W, Tper, s):
    G = L.global_frames(T, Tper, s)
    return G | set(range(max(0, t - W), min(T, t + W + 1)))


def _fixed_globals(t, T, W, Tper, s):
    A, _, _ = L.attended_frames(t, T, W, Tper, 0)      # ignores the rotation
    return A


def _target_without_clip(t, T, W, Tper, s):
    # expands towards 2W+1 window frames beyond the globals but never stops at T
    G = L.global_frames(T, Tper, s)
    lo, hi = max(0, t - W), min(T - 1, t + W)
    while len(G | set(range(lo, hi + 1))) < len(G) + 2 * W + 1 and (lo > 0 or hi < T - 1):
        if lo > 0:
            lo -= 1
        else:
            hi += 1
    return G | set(range(lo, hi + 1))


@pytest.mark.parametrize("bad", [_no_expansion, _fixed_globals, _target_without_clip])
def test_planted_mask_mistakes_are_caught(bad):
    failures = 0
    for (T, W, Tper, s, t), want in _golden():
        if sorted(bad(t, T, W, Tper, s)) != want:
            failures += 1
    uniform = all(len(bad(t, T, W, Tper, s)) == L.target_count(T, W, Tper, s)
                  for T, W, Tper, s in _sweep() for t in range(T))
    assert failures > 0 or not uniform
