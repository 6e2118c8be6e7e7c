"""fp64 CPU oracle: GSRS precise block importance and the attention-recall diagnostic.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA product path
never imports this module, and this module imports nothing from it.

Sources ("Sparse Attention for Video Generation Acceleration via Growing
Sparsity and Reduced Search", cited as GSRS):
  [GSRS §5.3]  the importance of key block j for query block i is the average
               attention weight that the query tokens of i give to the keys of
               j; over the key blocks of one query block it sums to one.
  [GSRS §5.3, §A.3] it is recovered exactly from per-block log-sum-exp
               statistics recorded during the attention pass, normalised with
               each row's own log-sum-exp (not a cached one).
  [GSRS §A.2]  when only some key blocks are evaluated, the weights are
               normalised over the evaluated key tokens and still sum to one.
  [GSRS §3.2]  attention recall: the fraction of the total attention weight
               that the selected blocks capture.

The steps follow that order: (1) per query row and evaluated key block, the
log-sum-exp of the row's scaled logits over the block's valid keys; (2) the
row's log-sum-exp over all evaluated keys; (3) exp((1) - (2)) averaged over
the valid rows of the query block.

Readings of points the pages leave open (each one is listed in the design notes):
  * rows of a query block are its valid tokens only (pad rows excluded); the
    keys of a key block are its valid tokens only.
  * logits are scale * q.k with the attention scale, in the permuted layout.
  * recall of a mask under the current attention is the sum, over the mask's
    blocks, of the importance evaluated with every key block (the dense
    attention's block weights); it is reported per query block.
  * importance of a key block outside the evaluated set is 0.
"""

from __future__ import annotations

import numpy as np

from .fvattn_oracle import num_blocks


def _valid_range(j: int, N: int, bs: int) -> tuple[int, int]:
    return j * bs, min((j + 1) * bs, N)


def block_lse_rows(qp, kp, mask_row, N: int, bs: int, scale: float, i: int) -> np.ndarray:
    """Step (1) for query block ``i`` of one head: ``[rows, nb]`` fp64.

    Entry (r, j) is log sum over the valid keys c of block j of
    exp(scale * q_r . k_c) for the valid query rows r of block i, for every
    evaluated block j (mask_row[j] true); -inf elsewhere.
    """
    qp = np.asarray(qp, np.float64)
    kp = np.asarray(kp, np.float64)
    nb = num_blocks(N, bs)
    lo, hi = _valid_range(i, N, bs)
    out = np.full((hi - lo, nb), -np.inf)
    for j in np.nonzero(np.asarray(mask_row))[0]:
        klo, khi = _valid_range(int(j), N, bs)
        logits = (qp[lo:hi] @ kp[klo:khi].T) * scale
        m = logits.max(axis=1)
        out[:, j] = m + np.log(np.exp(logits - m[:, None]).sum(axis=1))
    return out


def row_lse(blse_rows: np.ndarray) -> np.ndarray:
    """Step (2): the row's log-sum-exp over all evaluated keys, from its block values."""
    m = blse_rows.max(axis=1)
    return m + np.log(np.exp(blse_rows - m[:, None]).sum(axis=1))


def block_importance_row(qp, kp, mask_row, N: int, bs: int, scale: float, i: int) -> np.ndarray:
    """Step (3) for query block ``i`` of one head: importance over key blocks, ``[nb]``."""
    blse = block_lse_rows(qp, kp, mask_row, N, bs, scale, i)
    lse = row_lse(blse)
    return np.exp(blse - lse[:, None]).mean(axis=0)


def block_importance(qp, kp, mask, N: int, bs: int, scale: float, blocks=None) -> np.ndarray:
    """Importance of every (query block, key block) pair over ``[B, H, Npad, d]`` tensors.

    ``mask`` [B, H, nb, nb] bool is the evaluated set per query block (all
    blocks for the dense evaluation). Returns fp64 [B, H, nb, nb]; query
    blocks not listed in ``blocks`` (iterable of (b, h, i); all when None) are
    left at zero.
    """
    B, H = qp.shape[:2]
    nb = num_blocks(N, bs)
    out = np.zeros((B, H, nb, nb))
    todo = blocks if blocks is not None else [(b, h, i) for b in range(B) for h in range(H) for i in range(nb)]
    for (b, h, i) in todo:
        out[b, h, i] = block_importance_row(qp[b, h], kp[b, h], mask[b, h, i], N, bs, scale, i)
    return out


def attention_recall(importance_dense: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """Recall of ``mask`` [.., nb, nb] under the dense importance: per query block, ``[.., nb]``."""
    return np.where(np.asarray(mask, bool), importance_dense, 0.0).sum(axis=-1)
