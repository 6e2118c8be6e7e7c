"""The mask parity rule on hand-made cases (no GPU): an exact match passes, a flip at
the cut score counts as near_cut, a one-block count change at a cumulative sum on p
counts as count_flip, any other difference is hard, and the ceiling scales with the
selected pairs."""

import numpy as np

import oracle as O
from oracle.mask_parity import borderline_ceiling, summary
from parity import assert_mask_parity, compare_masks


def _orc(rows, p, k_min=1):
    s = np.asarray(rows, dtype=np.float64)
    order = np.empty(s.shape, dtype=np.int64)
    cnt = np.empty(s.shape[:-1], dtype=np.int64)
    for r in np.ndindex(*cnt.shape):
        order[r], cnt[r] = O.topp_topk_select(s[r], p, k_min)
    return {"scores": s, "order": order, "cnt": cnt}


def test_exact_match_has_no_mismatch():
    orc = _orc([[0.5, 0.3, 0.15, 0.05], [0.25, 0.25, 0.25, 0.25]], 0.7)
    mask = O.selection_mask(orc["order"], orc["cnt"])
    res = compare_masks(mask, orc, 0.7)
    assert res["mismatched"] == 0 and res["borderline"] == 0 and not res["hard"]
    assert res["rows"] == 2 and res["selected_pairs"] == int(mask.sum())


def test_tie_at_the_cut_is_near_cut():
    # blocks 1 and 2 tie at the cut score: choosing 2 instead of 1 is a legitimate fp32 outcome
    orc = _orc([[0.4, 0.2, 0.2, 0.2]], 0.55)
    mask = O.selection_mask(orc["order"], orc["cnt"])
    assert mask[0].tolist() == [True, True, False, False]
    mask[0, 1], mask[0, 2] = False, True
    res = compare_masks(mask, orc, 0.55)
    assert res["mismatched"] == 2 and res["near_cut"] == 2 and res["count_flip"] == 0 and not res["hard"]


def test_one_more_block_at_a_cumulative_sum_on_p_is_a_count_flip():
    # the first two blocks reach exactly p; an fp32 sum a hair below p takes the third
    orc = _orc([[0.5, 0.25, 0.15, 0.1]], 0.75)
    mask = O.selection_mask(orc["order"], orc["cnt"])
    assert mask[0].tolist() == [True, True, False, False]
    mask[0, 2] = True
    res = compare_masks(mask, orc, 0.75)
    assert res["mismatched"] == 1 and res["count_flip"] == 1 and res["near_cut"] == 0 and not res["hard"]


def test_any_other_difference_is_hard():
    orc = _orc([[0.5, 0.25, 0.15, 0.1]], 0.6)
    mask = O.selection_mask(orc["order"], orc["cnt"])
    mask[0, 3] = True                       # far below the cut, cumulative mass far from p
    res = compare_masks(mask, orc, 0.6)
    assert len(res["hard"]) == 1 and res["hard"][0][1] == 3
    mask = O.selection_mask(orc["order"], orc["cnt"])
    mask[0, 0] = False                      # the top block dropped
    res = compare_masks(mask, orc, 0.6)
    assert len(res["hard"]) == 1 and res["hard"][0][1] == 0


def test_ceiling_and_assertion():
    assert borderline_ceiling(0) == 1 and borderline_ceiling(10_000) == 1
    assert borderline_ceiling(10_001) == 2 and borderline_ceiling(1_000_000) == 100
    orc = _orc([[0.4, 0.2, 0.2, 0.2]] * 3, 0.55)
    mask = O.selection_mask(orc["order"], orc["cnt"])
    mask[0, 1], mask[0, 2] = False, True
    res = compare_masks(mask, orc, 0.55)
    try:
        assert_mask_parity(res, "two exempt blocks over a ceiling of one")
    except AssertionError as e:
        assert "near_cut=2" in str(e)
    else:
        raise AssertionError("the ceiling was not enforced")
    s = summary(res)
    assert s["hard"] == 0 and s["borderline"] == 2 and s["borderline_ceiling"] == 1
