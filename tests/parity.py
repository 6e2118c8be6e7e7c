"""Comparison helpers for GPU-vs-oracle parity tests (test infrastructure).

Mask rule (``oracle.mask_parity``): the GPU's selected set must equal the
oracle's for every query block, except for blocks on the Top-p cut. A
mismatched block is exempt when its oracle score is within 1e-5 (relative) of
the oracle's cut score s_(cnt-1) ("near_cut"), or, failing that, when the
oracle's cumulative importance of the blocks ranked before it is within 1e-5
of p ("count_flip", a one-block change of the count). Every other mismatch
fails, and the exempt blocks may not exceed 1e-4 of the selected pairs (at
least one): ``assert_mask_parity`` checks both and puts the counts in its
assertion message.
"""

from __future__ import annotations

import numpy as np

from oracle.mask_parity import BORDER_CUM, BORDER_REL, borderline_ceiling, mask_from_lists  # noqa: F401
from oracle.mask_parity import compare_masks as _compare
from oracle.fvattn_oracle import permute as _permute, tile_order as _tile_order

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
FP32_MAX_ABS = 1e-5


def check_lists_valid(kv_idx: np.ndarray, kv_cnt: np.ndarray, nb: int, k_min: int):
    """Structure every routed row must have: counts in range, ascending distinct in-range lists."""
    assert kv_cnt.min() >= min(k_min, nb) and kv_cnt.max() <= nb
    for row in np.ndindex(*kv_cnt.shape):
        c = int(kv_cnt[row])
        lst = kv_idx[row][:c]
        assert lst.min() >= 0 and lst.max() < nb, row
        assert np.all(np.diff(lst) > 0), row


def compare_masks(gpu_mask: np.ndarray, orc: dict, p: float) -> dict:
    """The counts of the mask rule (see ``oracle.mask_parity.compare_masks``)."""
    return _compare(gpu_mask, orc, p)


def mask_report(res: dict, label: str) -> str:
    return (f"{label}: rows={res['rows']} selected={res['selected_pairs']} mismatched={res['mismatched']} "
            f"near_cut={res['near_cut']} count_flip={res['count_flip']} hard={len(res['hard'])} "
            f"(ceiling {borderline_ceiling(res['selected_pairs'])})")


def assert_mask_parity(res: dict, label: str) -> str:
    """No hard mismatch, and the exempt blocks stay under the ceiling."""
    msg = mask_report(res, label)
    print(msg)
    assert not res["hard"], msg + f"; first failures {res['hard'][:5]}"
    ceiling = borderline_ceiling(res["selected_pairs"])
    assert res["borderline"] <= ceiling, msg
    assert res["count_flip"] <= ceiling, msg
    return msg


def attention_errors(gpu: np.ndarray, ref: np.ndarray):
    err = np.abs(gpu.astype(np.float64) - ref)
    return float(err.max()), float(err.mean())


def oracle_permuted(w, *tensors):
    """The seeded inputs in the oracle's own 3-D tile order, padded to nb*bs: the oracle's
    inputs never come from the library's permutation."""
    perm = _tile_order(*w.grid, *w.tile)
    return tuple(_permute(t.detach().float().cpu().numpy(), perm, w.block) for t in tensors)
