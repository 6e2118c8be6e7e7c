"""Mask parity rule: a routed block mask against the oracle's, block by block.

TEST INFRASTRUCTURE ONLY (see the package docstring): used by ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of ``bench.py`` to
compare a mask produced elsewhere with the oracle's routing result. It holds
no step of the method itself; the selection it checks against is
``topp_topk_select`` [FVAttn §2.1, §3.1; GSRS §5.2, §A.4].

The rule. The selected set must equal the oracle's for every query block,
except where the Top-p cut is numerically ambiguous. A GPU computes the block
scores and their cumulative sum in fp32, the oracle in fp64, so a block whose
score sits on the cut can legitimately fall on either side. A mismatched block
j of a row is exempt (counted, reported, not failed) when:

  * near_cut:   its oracle score is within BORDER_REL (relative) of the
                oracle's cut score s_(cnt-1), the smallest selected score; or
  * count_flip: it is not near the cut score, but the oracle's cumulative
                importance of the blocks ranked before it is within BORDER_CUM
                of p, so a one-ulp difference in the running sum moves the
                count by one (the GPU takes one block more or one fewer).

Every other mismatch is ``hard`` and fails. Both exemptions are counted
separately so that a report shows how often each one was used.
"""

from __future__ import annotations

import numpy as np

from .fvattn_oracle import selection_mask

BORDER_REL = 1e-5
BORDER_CUM = 1e-5


def mask_from_lists(kv_idx: np.ndarray, kv_cnt: np.ndarray, nb: int) -> np.ndarray:
    """Boolean [..., nb, nb] mask from index lists (entries [0, cnt) of each row)."""
    valid = np.arange(kv_idx.shape[-1]) < kv_cnt[..., None]
    mask = np.zeros(kv_idx.shape[:-1] + (nb,), dtype=bool)
    rows = np.nonzero(valid)
    mask[rows[:-1] + (kv_idx[valid],)] = True
    return mask


def compare_masks(gpu_mask: np.ndarray, orc: dict, p: float) -> dict:
    """Compare a boolean mask [..., nb, nb] with the oracle routing result ``orc``
    (the dict of ``route``: scores, order, cnt). Returns a dict:

      rows            query blocks compared
      selected_pairs  (query block, key block) pairs the oracle selects
      mismatched      blocks whose membership differs
      near_cut        mismatches exempt by the cut-score clause
      count_flip      mismatches exempt only by the cumulative-sum clause
      borderline      near_cut + count_flip
      hard            list of failing (row, j, score, cut score, mass before j)
    """
    omask = selection_mask(orc["order"], orc["cnt"])
    if gpu_mask.shape != omask.shape:
        raise ValueError(f"mask shape {gpu_mask.shape} != oracle {omask.shape}")
    diff = gpu_mask != omask
    res = {"rows": int(np.prod(omask.shape[:-1])), "selected_pairs": int(omask.sum()),
           "mismatched": int(diff.sum()), "near_cut": 0, "count_flip": 0, "borderline": 0, "hard": []}
    if res["mismatched"] == 0:
        return res
    for row in zip(*np.nonzero(diff.any(axis=-1))):
        s = orc["scores"][row]
        order = orc["order"][row]
        cnt = int(orc["cnt"][row])
        rank = np.empty_like(order)
        rank[order] = np.arange(len(order))
        cum = np.concatenate([[0.0], np.cumsum(s[order])])     # cum[r] = mass ranked before r
        s_cut = s[order[cnt - 1]]
        for j in np.nonzero(diff[row])[0]:
            if abs(s[j] - s_cut) <= BORDER_REL * s_cut:
                res["near_cut"] += 1
            elif abs(cum[rank[j]] - p) <= BORDER_CUM:
                res["count_flip"] += 1
            else:
                res["hard"].append((tuple(int(x) for x in row), int(j), float(s[j]), float(s_cut),
                                    float(cum[rank[j]])))
    res["borderline"] = res["near_cut"] + res["count_flip"]
    return res


def borderline_ceiling(selected_pairs: int, frac: float = 1e-4) -> int:
    """Largest number of exempt blocks accepted for a mask of ``selected_pairs``
    pairs: ``frac`` of them, at least one. A kernel that mis-selected blocks near
    the cut on a sizeable fraction of rows exceeds it."""
    return max(1, int(np.ceil(frac * selected_pairs)))


def summary(res: dict) -> dict:
    """The counts of ``compare_masks`` without the (possibly long) list of failures."""
    out = {k: v for k, v in res.items() if k != "hard"}
    out["hard"] = len(res["hard"])
    out["borderline_ceiling"] = borderline_ceiling(res["selected_pairs"])
    return out
