"""GPU parity of the GSRS diagnostic: block log-sum-exps recorded by the attention
kernels, exact block importance and attention recall, through the C-ABI, against
the fp64 oracle run on the GPU's own mask.

Tolerances, from the arithmetic:
  * block_lse. The logits are exact products of bf16 values summed in fp32
    (relative error ~1e-6 of |s|). The exponentials are ex2.approx of fp32
    arguments |x| <= ~40 (abs. error ~5e-6 in x), summed in fp32 over at most
    128 keys (~1e-5 relative), and the log is lg2.approx. So
    |error| <= ~2e-5 + 1e-6 |lse|. The gate is 2e-4 absolute.
  * importance. It is a mean of exp(block_lse - lse), each argument off by at
    most 4e-4, so the relative error is <= 4e-4. The gate is 5e-5 + 5e-4 * value.
    Entries outside the evaluated set are exactly 0, and each row sums to 1
    within 1e-4.
  * recall. It sums at most nb importances of one dense row, which themselves
    sum to 1 within 1e-4, so the gate is 1e-3 absolute.
The SIMT kernel (fp32 or d = 64) uses expf/logf and meets the same gates with room.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import mask_from_lists, oracle_permuted
from test_gpu_parity import BS64, ODD, ODD128, PEAKY, _np, _route_gpu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_video_b200 as F

BLSE_ABS = 2e-4
IMP_ABS, IMP_REL = 5e-5, 5e-4
RECALL_ABS = 1e-3
SENTINEL = 12345.0


def _diag_gpu(w, qp, kp, vp, kv_idx=None, kv_cnt=None):
    """One attention call with lse and block_lse, then importance. Returns numpy arrays."""
    dev = qp.device
    nb = O.num_blocks(w.N, w.block)
    op = torch.empty_like(qp)
    lse = torch.empty(qp.shape[:-1], dtype=torch.float32, device=dev)
    blse = torch.full((w.B, w.H, nb, qp.shape[2]), SENTINEL, dtype=torch.float32, device=dev)
    opk = F.FVATTN_OP_DENSE_FWD if kv_idx is None else F.FVATTN_OP_SPARSE_FWD
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(opk, w.B, w.H, w.N, w.d, w.block), dev)
    if kv_idx is None:
        F.fvattn_dense_fwd(qp, kp, vp, op, w.N, w.block, ws, lse=lse, block_lse=blse)
    else:
        F.fvattn_sparse_fwd(qp, kp, vp, op, kv_idx, kv_cnt, w.N, w.block, ws, lse=lse, block_lse=blse)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    imp = torch.full((w.B, w.H, nb, nb), float("nan"), dtype=torch.float32, device=dev)
    wsd = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_DIAG, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_block_importance(blse, lse, imp, w.N, w.block, wsd, kv_idx=kv_idx, kv_cnt=kv_cnt)
    assert F.fvattn_workspace_status(wsd) == F.FVATTN_OK
    return blse.cpu().numpy(), lse.cpu().numpy(), imp.cpu().numpy()


def _recall_gpu(w, imp_dense, kv_idx, kv_cnt):
    dev = kv_idx.device
    nb = O.num_blocks(w.N, w.block)
    rec = torch.full((w.B, w.H, nb), float("nan"), dtype=torch.float32, device=dev)
    wsd = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_DIAG, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_attention_recall(torch.from_numpy(imp_dense).to(dev), kv_idx, kv_cnt, rec, w.N, w.block, wsd)
    assert F.fvattn_workspace_status(wsd) == F.FVATTN_OK
    return rec.cpu().numpy()


def _check_rows(w, qn, kn, mask, blse, imp, rows):
    """Compare block_lse (evaluated pairs, valid rows) and importance rows with the oracle."""
    scale = 1.0 / math.sqrt(w.d)
    worst_b, worst_i = 0.0, 0.0
    for (b, h, i) in rows:
        ref_b = O.block_lse_rows(qn[b, h], kn[b, h], mask[b, h, i], w.N, w.block, scale, i)
        lo = i * w.block
        got_b = blse[b, h, :, lo:lo + ref_b.shape[0]].T           # [rows, nb]
        sel = mask[b, h, i]
        err_b = np.abs(got_b[:, sel] - ref_b[:, sel])
        worst_b = max(worst_b, float(err_b.max()))
        assert err_b.max() <= BLSE_ABS, (b, h, i, float(err_b.max()))
        # pairs outside the list are not written
        assert np.all(got_b[:, ~sel] == SENTINEL), (b, h, i)
        ref_i = np.exp(ref_b - O.row_lse(ref_b)[:, None]).mean(axis=0)
        ref_i[~sel] = 0.0
        err_i = np.abs(imp[b, h, i] - ref_i)
        worst_i = max(worst_i, float(err_i.max()))
        assert np.all(err_i <= IMP_ABS + IMP_REL * ref_i), (b, h, i, float(err_i.max()))
        assert np.all(imp[b, h, i][~sel] == 0.0)
        assert abs(float(imp[b, h, i].sum()) - 1.0) <= 1e-4
    return worst_b, worst_i


@pytest.mark.parametrize("w", [S.WORKLOADS["tiny"], ODD, ODD128, BS64, PEAKY], ids=lambda w: w.name)
def test_sparse_block_lse_and_importance_match_oracle(w):
    q, k, v = S.make_qkv(w, device="cuda")
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    vp = torch.empty_like(qp)
    F.fvattn_permute(v, vp, grid)
    blse, _, imp = _diag_gpu(w, qp, kp, vp, kv_idx, kv_cnt)
    mask = mask_from_lists(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), grid.nb)
    qn, kn = oracle_permuted(w, q, k)   # the oracle's own tile order of the seeded inputs
    rows = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(grid.nb)]
    wb, wi = _check_rows(w, qn, kn, mask, blse, imp, rows)
    print(f"{w.name}: density {mask.mean():.3f} max |d block_lse| {wb:.2e} max |d importance| {wi:.2e}")


@pytest.mark.parametrize("w", [S.WORKLOADS["tiny"], ODD128, BS64], ids=lambda w: w.name)
def test_dense_importance_and_recall_of_routed_mask(w):
    q, k, v = S.make_qkv(w, device="cuda")
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    vp = torch.empty_like(qp)
    F.fvattn_permute(v, vp, grid)
    nb = grid.nb
    blse, _, imp = _diag_gpu(w, qp, kp, vp)
    full = np.ones((w.B, w.H, nb, nb), bool)
    qn, kn = oracle_permuted(w, q, k)   # the oracle's own tile order of the seeded inputs
    rows = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(nb)]
    _check_rows(w, qn, kn, full, blse, imp, rows)
    rec = _recall_gpu(w, imp, kv_idx, kv_cnt)
    mask = mask_from_lists(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), nb)
    ref_imp = O.block_importance(qn, kn, full, w.N, w.block, 1.0 / math.sqrt(w.d))
    ref_rec = O.attention_recall(ref_imp, mask)
    assert np.abs(rec - ref_rec).max() <= RECALL_ABS
    # a full list recalls everything
    all_idx = torch.arange(nb, dtype=torch.int32, device="cuda").expand(w.B, w.H, nb, nb).contiguous()
    all_cnt = torch.full((w.B, w.H, nb), nb, dtype=torch.int32, device="cuda")
    assert np.abs(_recall_gpu(w, imp, all_idx, all_cnt) - 1.0).max() <= 1e-4
    print(f"{w.name}: mean recall of the routed mask {rec.mean():.4f} (oracle {ref_rec.mean():.4f})")


def test_importance_and_recall_sampled_480p():
    # full 1.3B-480p call (12 heads, 256 blocks), oracle on sampled query blocks
    w = S.WORKLOADS["wan1.3b-480p"]
    q, k, v = S.make_qkv(w, device="cuda")
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    vp = torch.empty_like(qp)
    F.fvattn_permute(v, vp, grid)
    nb = grid.nb
    blse, _, imp = _diag_gpu(w, qp, kp, vp, kv_idx, kv_cnt)
    mask = mask_from_lists(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), nb)
    rng = np.random.default_rng(5)
    rows = [(0, int(h), int(i)) for h, i in zip(rng.integers(0, w.H, 12), rng.integers(0, nb, 12))]
    rows.append((0, w.H - 1, nb - 1))               # the ragged last block
    qn, kn = oracle_permuted(w, q, k)   # the oracle's own tile order of the seeded inputs
    _check_rows(w, qn, kn, mask, blse, imp, rows)
    imp_gpu = torch.from_numpy(imp)
    sums = imp_gpu.sum(-1)
    assert float((sums - 1).abs().max()) <= 1e-4
    # dense evaluation and the recall of the routed mask, checked on the same rows
    dblse, _, dimp = _diag_gpu(w, qp, kp, vp)
    rec = _recall_gpu(w, dimp, kv_idx, kv_cnt)
    full = np.ones(nb, bool)
    scale = 1.0 / math.sqrt(w.d)
    for (b, h, i) in rows:
        ref = O.block_importance_row(qn[b, h], kn[b, h], full, w.N, w.block, scale, i)
        assert np.all(np.abs(dimp[b, h, i] - ref) <= IMP_ABS + IMP_REL * ref)
        assert abs(rec[b, h, i] - float(O.attention_recall(ref, mask[b, h, i]))) <= RECALL_ABS
    print(f"wan1.3b-480p: mean recall of the routed mask {rec.mean():.4f}, "
          f"min {rec.min():.4f}, density {mask.mean():.3f}")


def _select_gpu(w, imp_t, p, k_min):
    dev = imp_t.device
    nb = imp_t.shape[-1]
    idx = torch.full((w.B, w.H, nb, nb), -1, dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.H, nb), dtype=torch.int32, device=dev)
    hw = torch.empty((w.B, w.H), dtype=torch.int64, device=dev)
    wsd = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_DIAG, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_select_topp(imp_t, w.N, w.block, p, k_min, idx, cnt, hw, wsd)
    assert F.fvattn_workspace_status(wsd) == F.FVATTN_OK
    return idx.cpu().numpy(), cnt.cpu().numpy(), hw.cpu().numpy()


@pytest.mark.parametrize("w", [ODD128, BS64], ids=lambda w: w.name)
@pytest.mark.parametrize("p,k_min", [(0.8, 2), (0.5, 1), (1.0, 1)])
def test_select_topp_on_importance_matches_oracle(w, p, k_min):
    from parity import assert_mask_parity, check_lists_valid, compare_masks
    q, k, v = S.make_qkv(w, device="cuda")
    grid, qp, kp, _, _, _ = _route_gpu(w, q, k)
    vp = torch.empty_like(qp)
    F.fvattn_permute(v, vp, grid)
    _, _, imp = _diag_gpu(w, qp, kp, vp)                     # dense importance, fp32
    idx, cnt, hw = _select_gpu(w, torch.from_numpy(imp).cuda(), p, k_min)
    nb = grid.nb
    check_lists_valid(idx, cnt, nb, k_min)
    assert np.array_equal(hw, cnt.astype(np.int64).sum(-1))
    scores = imp.astype(np.float64)
    order = np.empty(scores.shape, dtype=np.int64)
    ocnt = np.empty(scores.shape[:-1], dtype=np.int64)
    for row in np.ndindex(*ocnt.shape):
        order[row], ocnt[row] = O.topp_topk_select(scores[row], p, k_min)
    assert_mask_parity(compare_masks(mask_from_lists(idx, cnt, nb),
                                     {"scores": scores, "order": order, "cnt": ocnt}, p),
                       f"{w.name} p={p} k_min={k_min}")


def test_gsrs_search_over_candidates():
    # candidates from the router, exact importance over them, then a tighter Top-p inside them
    w = ODD128
    q, k, v = S.make_qkv(w, device="cuda")
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    vp = torch.empty_like(qp)
    F.fvattn_permute(v, vp, grid)
    _, _, imp = _diag_gpu(w, qp, kp, vp, kv_idx, kv_cnt)      # normalised over the candidates
    nb = grid.nb
    cand = mask_from_lists(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), nb)
    idx, cnt, _ = _select_gpu(w, torch.from_numpy(imp).cuda(), 0.8, 1)
    sel = mask_from_lists(idx, cnt, nb)
    assert np.all(sel <= cand)                                   # inside the candidate set
    mass = np.where(sel, imp, 0.0).sum(-1)
    assert np.all(mass >= 0.8 - 1e-5)                            # covers p of the candidates' mass
    smallest = np.where(sel, imp, np.inf).min(-1)
    assert np.all((cnt == 1) | (mass - smallest < 0.8 + 1e-5))   # minimal prefix
    print(f"search: candidates density {cand.mean():.3f} -> {sel.mean():.3f}")
