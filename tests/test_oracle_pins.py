"""Pins of the fp64 oracle against what the pages and the mathematics fix.

No GPU. Each oracle function is checked against something other than itself:
hand-derived fixtures under tests/golden/, closed forms, invariants, brute
force on tiny inputs, and an independent library implementation (torch SDPA in
fp64) for textbook attention. The last section plants plausible mistakes in
copies of oracle steps and shows that a pin catches each of them.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_tile_golden():
    cases = []
    with open(os.path.join(GOLDEN, "tile_order.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, tail = line.split(":")
            cases.append((tuple(int(v) for v in head.split()), [int(v) for v in tail.split()]))
    return cases


def _read_topp_golden():
    rows = []
    with open(os.path.join(GOLDEN, "topp_rows.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            s, p, k, cnt, sel = [part.strip() for part in line.split("|")]
            rows.append((np.array([float(v) for v in s.split()]), float(p), int(k), int(cnt),
                         sorted(int(v) for v in sel.split())))
    return rows


# ----------------------------------------------------------------------------
# Step 1: tile permutation
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("case", _read_tile_golden())
def test_tile_order_golden(case):
    (T, Hh, W, tt, th, tw), expected = case
    assert O.tile_order(T, Hh, W, tt, th, tw).tolist() == expected


def _tile_order_nested(T, Hh, W, tt, th, tw):
    """Independent construction: walk tiles in raster order, then their tokens."""
    out = []
    for t0 in range(0, T, tt):
        for y0 in range(0, Hh, th):
            for x0 in range(0, W, tw):
                for t in range(t0, min(t0 + tt, T)):
                    for y in range(y0, min(y0 + th, Hh)):
                        for x in range(x0, min(x0 + tw, W)):
                            out.append((t * Hh + y) * W + x)
    return out


@pytest.mark.parametrize("grid", [(4, 8, 8, 1, 8, 8), (5, 7, 9, 2, 3, 4), (21, 30, 52, 2, 8, 8),
                                  (3, 5, 6, 1, 1, 1), (2, 9, 11, 3, 4, 5)])
def test_tile_order_matches_nested_walk_and_is_bijection(grid):
    perm = O.tile_order(*grid)
    T, Hh, W = grid[:3]
    assert sorted(perm.tolist()) == list(range(T * Hh * W))
    assert perm.tolist() == _tile_order_nested(*grid)


def test_tile_order_unit_tiles_is_identity():
    assert O.tile_order(3, 4, 5, 1, 1, 1).tolist() == list(range(60))


def test_tile_order_full_tiles_are_contiguous_chunks():
    T, Hh, W, tt, th, tw = 4, 16, 24, 2, 8, 8
    perm = O.tile_order(T, Hh, W, tt, th, tw)
    size = tt * th * tw
    for c in range(len(perm) // size):
        chunk = perm[c * size:(c + 1) * size]
        t = chunk // (Hh * W)
        y = (chunk // W) % Hh
        x = chunk % W
        assert len(set((t // tt).tolist())) == 1
        assert len(set((y // th).tolist())) == 1
        assert len(set((x // tw).tolist())) == 1


def test_permute_inverse_roundtrip_and_padding():
    rng = np.random.default_rng(0)
    perm = O.tile_order(3, 5, 7, 2, 2, 4)           # N = 105, not a multiple of 16
    x = rng.standard_normal((2, 3, 105, 4))
    y = O.permute(x, perm, 16)
    assert y.shape == (2, 3, 112, 4)
    assert np.all(y[..., 105:, :] == 0)
    np.testing.assert_array_equal(y[..., 7, :], x[..., perm[7], :])
    np.testing.assert_array_equal(O.inverse_permute(y, perm), x)


def test_permute_golden_small():
    perm = np.array(_read_tile_golden()[1][1])      # T=3 Hh=2 W=2, tiles 2x2x1
    x = np.arange(12, dtype=np.float64).reshape(1, 1, 12, 1) * 10
    y = O.permute(x, perm, 8)
    assert y[0, 0, :, 0].tolist() == [0, 20, 40, 60, 10, 30, 50, 70, 80, 100, 90, 110, 0, 0, 0, 0]


# ----------------------------------------------------------------------------
# Step 2: pooling and block scores
# ----------------------------------------------------------------------------
def test_pool_golden_partial_last_block():
    xp = np.array([1.0, 2.0, 3.0, 4.0, 10.0, 0.0]).reshape(6, 1)   # N=5, bs=2, one pad row
    assert O.block_mean_pool(xp, 5, 2)[:, 0].tolist() == [1.5, 3.5, 10.0]


def test_pool_constant_blocks_and_ramp():
    bs, nb, d = 8, 5, 3
    N = bs * nb - 3
    vals = np.arange(nb * d, dtype=np.float64).reshape(nb, d) - 4.0
    xp = np.repeat(vals, bs, axis=0)
    xp[N:] = 123.0                                   # pad rows must not count
    np.testing.assert_array_equal(O.block_mean_pool(xp, N, bs), vals)
    ramp = np.arange(N + 3, dtype=np.float64).reshape(-1, 1)
    pooled = O.block_mean_pool(ramp, N, bs)[:, 0]
    mids = [(i * bs + min((i + 1) * bs, N) - 1) / 2 for i in range(nb)]   # mean of a run = midpoint
    np.testing.assert_allclose(pooled, mids, rtol=0, atol=1e-12)


def test_block_scores_closed_form_two_blocks():
    qbar = np.array([[1.0, 0.0]])
    kbar = np.array([[0.0, 0.0], [2.0, 0.0]])
    s = O.block_scores(qbar, kbar, 1.0 / math.sqrt(2.0))
    e = math.exp(2.0 / math.sqrt(2.0))
    np.testing.assert_allclose(s[0], [1.0 / (1.0 + e), e / (1.0 + e)], rtol=1e-15)


def test_block_scores_rows_sum_to_one_and_zero_query_is_uniform():
    rng = np.random.default_rng(1)
    qbar = rng.standard_normal((2, 7, 16)) * 3
    kbar = rng.standard_normal((2, 9, 16))
    s = O.block_scores(qbar, kbar, 0.25)
    np.testing.assert_allclose(s.sum(-1), 1.0, rtol=0, atol=1e-14)
    assert np.all(s > 0)
    s0 = O.block_scores(np.zeros((3, 16)), rng.standard_normal((4, 16)), 0.25)
    assert np.all(s0 == 0.25)                         # exact: exp(0)=1, 1/4 representable


def test_block_scores_large_logits_stay_finite():
    s = O.block_scores(np.array([[1000.0]]), np.array([[1.0], [0.5], [-2.0]]), 1.0)
    assert np.all(np.isfinite(s))
    np.testing.assert_allclose(s[0], [1.0, 0.0, 0.0], atol=1e-200)


# ----------------------------------------------------------------------------
# Step 3: Top-p with Top-k floor
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("row", _read_topp_golden())
def test_topp_golden_rows(row):
    s, p, k_min, cnt_exp, sel_exp = row
    order, cnt = O.topp_topk_select(s, p, k_min)
    assert cnt == cnt_exp
    assert sorted(order[:cnt].tolist()) == sel_exp


def _brute_force_select(s, p, k_min):
    """Enumerate subsets: the minimum-size subsets with mass >= p, the max-mass one
    (ties: the subset whose sorted index tuple is smallest); then the floor."""
    nbk = len(s)
    if p >= 1.0:
        return list(range(nbk))
    best = None
    for c in range(1, nbk + 1):
        cands = [S for S in itertools.combinations(range(nbk), c) if sum(s[j] for j in S) >= p]
        if cands:
            best = max(cands, key=lambda S: (sum(s[j] for j in S), [-j for j in S]))
            break
    if best is None:
        best = tuple(range(nbk))
    if len(best) < k_min:
        c = min(k_min, nbk)
        best = max(itertools.combinations(range(nbk), c),
                   key=lambda S: (sum(s[j] for j in S), [-j for j in S]))
    return sorted(best)


@pytest.mark.parametrize("seed", range(40))
def test_topp_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    nbk = int(rng.integers(2, 9))
    s = O.block_scores(rng.standard_normal((1, 4)) * rng.uniform(0.1, 3),
                       rng.standard_normal((nbk, 4)), 1.0)[0]
    for p in (0.3, 0.5, 0.8, 0.9, 0.95, 1.0):
        for k_min in (1, 2, 4):
            order, cnt = O.topp_topk_select(s, p, k_min)
            assert sorted(order[:cnt].tolist()) == _brute_force_select(s, p, k_min), (p, k_min)


@pytest.mark.parametrize("seed", range(10))
def test_topp_coverage_minimality_and_floor(seed):
    rng = np.random.default_rng(100 + seed)
    nbk = 57
    s = O.block_scores(rng.standard_normal((1, 8)) * 2, rng.standard_normal((nbk, 8)), 1.0)[0]
    for p in (0.5, 0.9, 0.95, 0.99):
        for k_min in (1, 4, 16, 60):
            order, cnt = O.topp_topk_select(s, p, k_min)
            ranked = s[order]
            assert ranked[:-1].tolist() == sorted(ranked.tolist(), reverse=True)[:-1]
            assert min(k_min, nbk) <= cnt <= nbk
            if cnt < nbk:
                assert ranked[:cnt].sum() >= p - 1e-12          # coverage
            if cnt > k_min:
                assert ranked[:cnt - 1].sum() < p               # minimality above the floor


def test_topp_p_one_and_large_floor_select_all():
    s = np.array([0.5, 0.2, 0.2, 0.1])
    assert O.topp_topk_select(s, 1.0, 1)[1] == 4
    assert O.topp_topk_select(s, 0.1, 4)[1] == 4
    assert O.topp_topk_select(s, 0.1, 99)[1] == 4


def test_selection_mask_and_head_work():
    order = np.array([[[2, 0, 1], [1, 2, 0], [0, 1, 2]]])
    cnt = np.array([[2, 1, 3]])
    m = O.selection_mask(order, cnt)
    assert m.tolist() == [[[True, False, True], [False, True, False], [True, True, True]]]
    assert O.head_work(cnt).tolist() == [6]
    assert m.sum(-1).tolist() == cnt.tolist()


def test_route_composes_steps_on_tiny():
    rng = np.random.default_rng(3)
    T, Hh, W = 4, 8, 8
    q = rng.standard_normal((1, 2, T * Hh * W, 16))
    k = rng.standard_normal((1, 2, T * Hh * W, 16))
    r = O.route(q, k, (T, Hh, W, 1, 8, 8), 64, 0.9, 1)
    assert r["cnt"].shape == (1, 2, 4)
    np.testing.assert_allclose(r["scores"].sum(-1), 1.0, atol=1e-14)
    # first tile = frame 0: pooled q of block 0 is the mean of frame 0's tokens
    np.testing.assert_allclose(r["qbar"][0, 0, 0], q[0, 0, :64].mean(0), atol=1e-14)
    assert r["head_work"].tolist() == [r["cnt"][0].sum(-1).tolist()]


# ----------------------------------------------------------------------------
# Step 4: attention
# ----------------------------------------------------------------------------
def test_dense_attention_closed_form():
    q = np.array([[[[1.0, 0.0]]]])
    k = np.array([[[[0.0, 0.0], [2.0, 0.0]]]])
    v = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])
    out = O.dense_attention(q, k, v, 1.0 / math.sqrt(2.0))
    e = math.exp(math.sqrt(2.0))
    np.testing.assert_allclose(out[0, 0, 0], [1 / (1 + e), e / (1 + e)], rtol=1e-15)


def test_dense_attention_matches_torch_sdpa_fp64():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((2, 3, 37, 16)) * 2
    k = rng.standard_normal((2, 3, 41, 16))
    v = rng.standard_normal((2, 3, 41, 16))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), scale=0.3).numpy()
    np.testing.assert_allclose(O.dense_attention(q, k, v, 0.3), ref, rtol=1e-12, atol=1e-13)


def _tiny_perm_inputs(seed, N_grid=(3, 5, 7), tile=(1, 4, 4), bs=32, d=8):
    rng = np.random.default_rng(seed)
    perm = O.tile_order(*N_grid, *tile)
    N = len(perm)
    x = [rng.standard_normal((1, 2, N, d)) for _ in range(3)]
    xp = [O.permute(t, perm, bs) for t in x]
    return perm, N, x, xp


def test_full_mask_equals_dense_attention():
    perm, N, (q, k, v), (qp, kp, vp) = _tiny_perm_inputs(5)
    bs = 32
    nb = O.num_blocks(N, bs)
    mask = np.ones((1, 2, nb, nb), dtype=bool)
    out = O.masked_attention(qp, kp, vp, mask, N, bs, 0.35)
    dense = O.dense_attention(q, k, v, 0.35)
    np.testing.assert_allclose(O.inverse_permute(out, perm), dense, rtol=1e-12, atol=1e-13)


def test_p_one_route_gives_dense_attention():
    perm, N, (q, k, v), (qp, kp, vp) = _tiny_perm_inputs(6)
    r = O.route(q, k, (3, 5, 7, 1, 4, 4), 32, 1.0, 1)
    mask = O.selection_mask(r["order"], r["cnt"])
    assert mask.all()
    out = O.masked_attention(qp, kp, vp, mask, N, 32, 0.35)
    np.testing.assert_allclose(O.inverse_permute(out, perm), O.dense_attention(q, k, v, 0.35),
                               rtol=1e-12, atol=1e-13)


def test_zero_query_gives_mean_of_selected_valid_values():
    perm, N, _, (qp, kp, vp) = _tiny_perm_inputs(7)
    bs = 32
    nb = O.num_blocks(N, bs)                                     # N=105 -> last block 9 valid
    mask = np.zeros((1, 2, nb, nb), dtype=bool)
    mask[0, 0, 1, [0, nb - 1]] = True
    qz = np.zeros_like(qp)
    rows = O.masked_attention_rows(qz[0, 0], kp[0, 0], vp[0, 0], mask[0, 0, 1], N, bs, 0.5, 1)
    keys = list(range(0, 32)) + list(range((nb - 1) * bs, N))
    np.testing.assert_allclose(rows, np.broadcast_to(vp[0, 0, keys].mean(0), rows.shape), atol=1e-14)


def test_single_block_equals_dense_on_that_block_and_single_key():
    perm, N, _, (qp, kp, vp) = _tiny_perm_inputs(8)
    bs = 32
    nb = O.num_blocks(N, bs)
    row = np.zeros(nb, dtype=bool)
    row[2] = True
    rows = O.masked_attention_rows(qp[0, 1], kp[0, 1], vp[0, 1], row, N, bs, 0.4, 0)
    ref = O.dense_attention(qp[0, 1, None, None, :32], kp[0, 1, None, None, 64:96],
                            vp[0, 1, None, None, 64:96], 0.4)[0, 0]
    np.testing.assert_allclose(rows, ref, rtol=1e-13, atol=1e-14)
    # a block with a single valid key returns that key's value row
    only_last = np.zeros(nb, dtype=bool)
    only_last[nb - 1] = True
    N1 = (nb - 1) * bs + 1
    rows = O.masked_attention_rows(qp[0, 0], kp[0, 0], vp[0, 0], only_last, N1, bs, 0.4, 0)
    np.testing.assert_allclose(rows, np.broadcast_to(vp[0, 0, N1 - 1], rows.shape), atol=1e-15)


def test_pad_keys_never_attended():
    perm, N, _, (qp, kp, vp) = _tiny_perm_inputs(9)
    bs = 32
    nb = O.num_blocks(N, bs)
    kp2, vp2 = kp.copy(), vp.copy()
    kp2[..., N:, :] = 50.0                                       # huge logits if attended
    vp2[..., N:, :] = 1e6
    row = np.ones(nb, dtype=bool)
    a = O.masked_attention_rows(qp[0, 0], kp[0, 0], vp[0, 0], row, N, bs, 0.4, 1)
    b = O.masked_attention_rows(qp[0, 0], kp2[0, 0], vp2[0, 0], row, N, bs, 0.4, 1)
    np.testing.assert_array_equal(a, b)


# ----------------------------------------------------------------------------
# Planted mistakes: a plausible slip in each step must fail a pin above.
# ----------------------------------------------------------------------------
def _tile_order_xy_swapped(T, Hh, W, tt, th, tw):
    keys = sorted(((t // tt, x // tw, y // th, t % tt, y % th, x % tw), (t * Hh + y) * W + x)
                  for t in range(T) for y in range(Hh) for x in range(W))
    return [n for _, n in keys]


def _pool_divides_by_bs(xp, N, bs):
    nb = O.num_blocks(N, bs)
    return np.array([xp[i * bs:min((i + 1) * bs, N)].sum(0) / bs for i in range(nb)])


def _topp_strict(s, p, k_min):
    order = np.lexsort((np.arange(len(s)), -s))
    cum = np.cumsum(s[order])
    hit = np.nonzero(cum > p)[0]
    n_p = int(hit[0]) + 1 if hit.size else len(s)
    return order, min(len(s), max(n_p, k_min))


def _topp_ties_high_first(s, p, k_min):
    order = np.lexsort((-np.arange(len(s)), -s))
    cum = np.cumsum(s[order])
    hit = np.nonzero(cum >= p)[0]
    n_p = int(hit[0]) + 1 if hit.size else len(s)
    return order, min(len(s), max(n_p, k_min))


def test_planted_mistakes_are_caught():
    (g1, exp1), _ = _read_tile_golden()
    assert _tile_order_xy_swapped(*g1) != exp1
    xp = np.array([1.0, 2.0, 3.0, 4.0, 10.0, 0.0]).reshape(6, 1)
    assert _pool_divides_by_bs(xp, 5, 2)[:, 0].tolist() != [1.5, 3.5, 10.0]
    rows = _read_topp_golden()
    strict_fail = any(sorted(_topp_strict(s, p, k)[0][:_topp_strict(s, p, k)[1]].tolist()) != sel
                      for s, p, k, c, sel in rows)
    ties_fail = any(sorted(_topp_ties_high_first(s, p, k)[0][:_topp_ties_high_first(s, p, k)[1]].tolist()) != sel
                    for s, p, k, c, sel in rows)
    assert strict_fail and ties_fail
    # a score step that forgets the 1/sqrt(d) temperature fails the closed form
    s_noscale = O.block_scores(np.array([[1.0, 0.0]]), np.array([[0.0, 0.0], [2.0, 0.0]]), 1.0)
    e = math.exp(2.0 / math.sqrt(2.0))
    assert not np.allclose(s_noscale[0], [1 / (1 + e), e / (1 + e)])
