"""Pins of the GSRS block-importance / attention-recall oracle (no GPU).

Each check ties the oracle to something other than itself:
  * the definition written a second way: the full attention matrix from
    torch.softmax (fp64, masked logits at -inf), summed over each key block's
    columns and averaged over each query block's rows;
  * closed forms: Q = 0 gives uniform attention over the evaluated keys, so a
    block's importance is its share of valid keys;
  * invariants from the pages: importance sums to one over the evaluated key
    blocks [GSRS §5.3, §A.2]; the block log-sum-exps combine to the row's
    log-sum-exp over all evaluated keys (checked against scipy's logsumexp);
    a Top-p selection made on the importance itself recalls at least p;
  * planted mistakes in copies of oracle steps, each caught by a pin above.
"""

import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O


def _qk(H, N, bs, d, seed, zero_q=False):
    rng = np.random.default_rng(seed)
    nb = O.num_blocks(N, bs)
    npad = nb * bs
    q = rng.standard_normal((1, H, npad, d))
    k = rng.standard_normal((1, H, npad, d))
    q[:, :, N:] = 0.0
    k[:, :, N:] = 0.0
    if zero_q:
        q[:] = 0.0
    return q * 1.5, k


def _random_mask(H, nb, seed, density=0.5):
    rng = np.random.default_rng(seed)
    m = rng.random((1, H, nb, nb)) < density
    m[..., 0] = True          # at least one evaluated block per row
    return m


def _explicit_importance(q, k, mask, N, bs, scale):
    """Importance through the full attention matrix (torch, fp64)."""
    B, H, npad, d = q.shape
    nb = O.num_blocks(N, bs)
    qt = torch.from_numpy(q[:, :, :N])
    kt = torch.from_numpy(k[:, :, :N])
    logits = torch.einsum("bhrd,bhcd->bhrc", qt, kt) * scale
    tok_blk = torch.arange(N) // bs
    keymask = torch.from_numpy(mask)[:, :, tok_blk][:, :, :, tok_blk]   # [B,H,N,N] query-token x key-token
    a = torch.softmax(logits.masked_fill(~keymask, float("-inf")), dim=-1)
    # column sums per key block, then row mean per query block
    per_blk = torch.zeros(B, H, N, nb, dtype=torch.float64).index_add_(3, tok_blk, a)
    out = torch.zeros(B, H, nb, nb, dtype=torch.float64).index_add_(2, tok_blk, per_blk)
    counts = torch.bincount(tok_blk, minlength=nb).to(torch.float64)
    return (out / counts[None, None, :, None]).numpy()


@pytest.mark.parametrize("N,bs", [(256, 64), (250, 64), (300, 128), (64, 64)])
def test_importance_equals_block_sums_of_the_attention_matrix(N, bs):
    H, d = 2, 16
    q, k = _qk(H, N, bs, d, seed=N)
    nb = O.num_blocks(N, bs)
    mask = _random_mask(H, nb, seed=N + 1)
    scale = 1.0 / math.sqrt(d)
    got = O.block_importance(q, k, mask, N, bs, scale)
    want = _explicit_importance(q, k, mask, N, bs, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("N,bs", [(300, 128), (200, 64)])
def test_importance_sums_to_one_over_evaluated_blocks(N, bs):
    H, d = 3, 32
    q, k = _qk(H, N, bs, d, seed=7)
    nb = O.num_blocks(N, bs)
    mask = _random_mask(H, nb, seed=8, density=0.4)
    imp = O.block_importance(q, k, mask, N, bs, 1.0 / math.sqrt(d))
    np.testing.assert_allclose(imp.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert np.all(imp[~mask] == 0.0)
    assert np.all(imp[mask] > 0.0)


def test_zero_query_gives_share_of_valid_keys():
    # uniform attention over the evaluated keys: importance of j = n_j / sum of n over the set
    N, bs, H, d = 250, 64, 2, 8            # last block holds 58 valid keys
    q, k = _qk(H, N, bs, d, seed=3, zero_q=True)
    nb = O.num_blocks(N, bs)
    mask = _random_mask(H, nb, seed=4)
    mask[0, 0, 1] = [True, False, True, True]
    imp = O.block_importance(q, k, mask, N, bs, 0.5)
    n = np.array([64, 64, 64, 58], dtype=np.float64)
    for h in range(H):
        for i in range(nb):
            want = np.where(mask[0, h, i], n, 0.0) / n[mask[0, h, i]].sum()
            np.testing.assert_allclose(imp[0, h, i], want, rtol=0, atol=1e-15)
    np.testing.assert_allclose(imp[0, 0, 1], [64 / 186, 0, 64 / 186, 58 / 186], rtol=0, atol=1e-15)


def test_block_lse_combines_to_row_lse():
    N, bs, H, d = 300, 128, 1, 32
    q, k = _qk(H, N, bs, d, seed=11)
    nb = O.num_blocks(N, bs)
    mask_row = np.array([True, False, True])
    scale = 1.0 / math.sqrt(d)
    for i in range(nb):
        blse = O.block_lse_rows(q[0, 0], k[0, 0], mask_row, N, bs, scale, i)
        lo, hi = i * bs, min((i + 1) * bs, N)
        cols = np.r_[0:128, 256:300]
        want = scipy.special.logsumexp((q[0, 0, lo:hi] @ k[0, 0, cols].T) * scale, axis=1)
        np.testing.assert_allclose(O.row_lse(blse), want, rtol=0, atol=1e-12)
        assert np.all(np.isneginf(blse[:, 1]))
        assert blse.shape == (hi - lo, nb)


def test_recall_of_full_mask_is_one_and_of_single_block_is_its_importance():
    N, bs, H, d = 300, 64, 2, 16
    q, k = _qk(H, N, bs, d, seed=21)
    nb = O.num_blocks(N, bs)
    full = np.ones((1, H, nb, nb), bool)
    imp = O.block_importance(q, k, full, N, bs, 0.25)
    np.testing.assert_allclose(O.attention_recall(imp, full), 1.0, rtol=0, atol=1e-12)
    one = np.zeros_like(full)
    one[..., 2] = True
    np.testing.assert_array_equal(O.attention_recall(imp, one), imp[..., 2])


@pytest.mark.parametrize("p", [0.5, 0.8, 0.95])
def test_topp_on_importance_recalls_at_least_p(p):
    # selecting by Top-p on the dense importance itself covers at least p of it
    N, bs, H, d = 640, 64, 2, 16
    q, k = _qk(H, N, bs, d, seed=31)
    nb = O.num_blocks(N, bs)
    full = np.ones((1, H, nb, nb), bool)
    imp = O.block_importance(q, k, full, N, bs, 0.6)
    for h in range(H):
        for i in range(nb):
            order, c = O.topp_topk_select(imp[0, h, i], p, 1)
            mask = np.zeros(nb, bool)
            mask[order[:c]] = True
            rec = float(O.attention_recall(imp[0, h, i], mask))
            assert rec >= p - 1e-12
            # minimality of the prefix: dropping the last selected block goes below p
            if c > 1:
                assert rec - imp[0, h, i, order[c - 1]] < p


# ---------------------------------------------------------------- planted mistakes

def _importance_pad_rows_counted(qp, kp, mask_row, N, bs, scale, i):
    blse = O.block_lse_rows(qp, kp, mask_row, N, bs, scale, i)
    lse = O.row_lse(blse)
    return np.exp(blse - lse[:, None]).sum(axis=0) / bs        # divides by bs, not by valid rows


def _importance_max_normalised(qp, kp, mask_row, N, bs, scale, i):
    blse = O.block_lse_rows(qp, kp, mask_row, N, bs, scale, i)
    return np.exp(blse - blse.max(axis=1, keepdims=True)).mean(axis=0)   # max, not the row LSE


def _importance_key_mean(qp, kp, mask_row, N, bs, scale, i):
    # averages the weights over a block's keys instead of summing them
    blse = O.block_lse_rows(qp, kp, mask_row, N, bs, scale, i)
    lse = O.row_lse(blse)
    nb = blse.shape[1]
    n = np.array([min(bs, N - j * bs) for j in range(nb)], dtype=np.float64)
    return (np.exp(blse - lse[:, None]) / n).mean(axis=0)


@pytest.mark.parametrize("bad", [_importance_pad_rows_counted, _importance_max_normalised,
                                 _importance_key_mean])
def test_planted_importance_mistakes_are_caught(bad):
    N, bs, H, d = 250, 64, 1, 16
    q, k = _qk(H, N, bs, d, seed=41)
    nb = O.num_blocks(N, bs)
    mask = _random_mask(H, nb, seed=42, density=0.7)
    scale = 0.25
    want = _explicit_importance(q, k, mask, N, bs, scale)
    got = np.stack([bad(q[0, 0], k[0, 0], mask[0, 0, i], N, bs, scale, i) for i in range(nb)])
    sums_ok = np.allclose(got.sum(-1), 1.0, atol=1e-9)
    matches = np.allclose(got, want[0, 0], atol=1e-9)
    assert not (sums_ok and matches)
