"""Comparison helpers for GPU-vs-oracle parity tests (test infrastructure).

Mask rule: the GPU's selected set must equal the oracle's for every query
block, except for blocks on the Top-p cut, which are counted as borderline:
a mismatched block j is borderline when its oracle score is within 1e-5
(relative) of the oracle's cut score s_(cnt-1), or when the oracle's
cumulative importance of the blocks ranked before j is within 1e-5 of p (a
count flip). Every other mismatch fails.
"""

from __future__ import annotations

import numpy as np

BORDER_REL = 1e-5
BORDER_CUM = 1e-5
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
FP32_MAX_ABS = 1e-5


def mask_from_lists(kv_idx: np.ndarray, kv_cnt: np.ndarray, nb: int) -> np.ndarray:
    """Boolean [..., nb, nb] mask from the ABI's lists (entries [0, cnt) per row)."""
    valid = np.arange(kv_idx.shape[-1]) < kv_cnt[..., None]
    mask = np.zeros(kv_idx.shape[:-1] + (nb,), dtype=bool)
    rows = np.nonzero(valid)
    mask[rows[:-1] + (kv_idx[valid],)] = True
    return mask


def check_lists_valid(kv_idx: np.ndarray, kv_cnt: np.ndarray, nb: int, k_min: int):
    """Structure every routed row must have: counts in range, ascending distinct in-range lists."""
    assert kv_cnt.min() >= min(k_min, nb) and kv_cnt.max() <= nb
    for row in np.ndindex(*kv_cnt.shape):
        c = int(kv_cnt[row])
        lst = kv_idx[row][:c]
        assert lst.min() >= 0 and lst.max() < nb, row
        assert np.all(np.diff(lst) > 0), row


def compare_masks(gpu_mask: np.ndarray, orc: dict, p: float):
    """Returns (n_mismatch, n_borderline, hard) with hard = list of failing (row, j)."""
    from oracle import selection_mask
    omask = selection_mask(orc["order"], orc["cnt"])
    diff = gpu_mask != omask
    n_mis = int(diff.sum())
    hard = []
    n_border = 0
    if n_mis == 0:
        return 0, 0, hard
    for row in zip(*np.nonzero(diff.any(axis=-1))):
        s = orc["scores"][row]
        order = orc["order"][row]
        cnt = int(orc["cnt"][row])
        rank = np.empty_like(order)
        rank[order] = np.arange(len(order))
        cum = np.concatenate([[0.0], np.cumsum(s[order])])     # cum[r] = mass ranked before r
        s_cut = s[order[cnt - 1]]
        for j in np.nonzero(diff[row])[0]:
            near_cut = abs(s[j] - s_cut) <= BORDER_REL * s_cut
            near_p = abs(cum[rank[j]] - p) <= BORDER_CUM
            if near_cut or near_p:
                n_border += 1
            else:
                hard.append((row, int(j), float(s[j]), float(s_cut), float(cum[rank[j]])))
    return n_mis, n_border, hard


def attention_errors(gpu: np.ndarray, ref: np.ndarray):
    err = np.abs(gpu.astype(np.float64) - ref)
    return float(err.max()), float(err.mean())
