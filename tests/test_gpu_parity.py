"""GPU parity: the CUDA path through the C-ABI against the fp64 oracle.

Masks are compared on every query block of every workload (borderline blocks
at the Top-p cut are counted, everything else must match bit for bit);
permutations bit-exactly; attention outputs against the oracle run on the
GPU's own mask (the gate: bf16 max-abs <= 2e-2 and mean-abs <= 2e-3, fp32
max-abs <= 1e-5), on every query block at the small sizes and on sampled
query blocks at the large ones.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import (BF16_MAX_ABS, BF16_MEAN_ABS, FP32_MAX_ABS, assert_mask_parity, attention_errors,
                    check_lists_valid, compare_masks, mask_from_lists, oracle_permuted)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_video_b200 as F


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


def _route_gpu(w, q, k):
    grid = F.Grid.make(w.grid, w.tile, w.block)
    dev = q.device
    nb, npad = grid.nb, grid.nb * w.block
    qp = torch.empty((w.B, w.H, npad, w.d), dtype=q.dtype, device=dev)
    kp = torch.empty_like(qp)
    kv_idx = torch.full((w.B, w.H, nb, nb), -7, dtype=torch.int32, device=dev)
    kv_cnt = torch.empty((w.B, w.H, nb), dtype=torch.int32, device=dev)
    hw = torch.empty((w.B, w.H), dtype=torch.int64, device=dev)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_route(q, k, grid, w.p, w.k_min, kv_idx, kv_cnt, hw, ws, qp_out=qp, kp_out=kp)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    return grid, qp, kp, kv_idx, kv_cnt, hw


def _attn_gpu(w, qp, kp, vp, kv_idx=None, kv_cnt=None, lse=False):
    dev = qp.device
    op = torch.full_like(qp, float("nan"))
    lse_t = torch.empty(qp.shape[:-1], dtype=torch.float32, device=dev) if lse else None
    opk = F.FVATTN_OP_DENSE_FWD if kv_idx is None else F.FVATTN_OP_SPARSE_FWD
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(opk, w.B, w.H, w.N, w.d, w.block), dev)
    if kv_idx is None:
        F.fvattn_dense_fwd(qp, kp, vp, op, w.N, w.block, ws, lse=lse_t)
    else:
        F.fvattn_sparse_fwd(qp, kp, vp, op, kv_idx, kv_cnt, w.N, w.block, ws, lse=lse_t)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    return op, lse_t


ODD = S.Workload("odd-grid", 2, 3, 64, "bf16", (5, 7, 9), (2, 3, 4), 64, 0.8, 2, seed=11)
ODD128 = S.Workload("odd-grid-128", 2, 3, 128, "bf16", (3, 10, 14), (2, 8, 8), 128, 0.85, 2, seed=12)
SINGLE = S.Workload("single-block", 1, 2, 128, "bf16", (1, 8, 10), (1, 8, 8), 128, 0.9, 1, seed=13)
TINY_BF16 = S.Workload("tiny-bf16-d128", 1, 2, 128, "bf16", (4, 16, 16), (1, 8, 16), 128, 0.9, 1,
                       seed=14, gen="gauss", peaky_head=1, peaky_scale=3.0)
# Large logits make the running max jump often, exercising the O rescale in TMEM.
PEAKY = S.Workload("peaky-rescale", 1, 3, 128, "bf16", (4, 16, 24), (1, 8, 16), 128, 0.97, 2,
                   seed=15, gen="gauss", peaky_head=2, peaky_scale=8.0)
BS64 = S.Workload("bs64-d128", 2, 2, 128, "bf16", (5, 12, 20), (1, 8, 8), 64, 0.8, 3, seed=16)
# 64-token blocks with an odd block count (the last unit's second block is past the end) and
# an odd number of units (3 heads x 9), so the last round of unit pairs has an idle slot
BS64_ODD = S.Workload("bs64-odd-units", 1, 3, 128, "bf16", (4, 16, 17), (1, 8, 8), 64, 0.7, 2, seed=19)
# d = 64 on the tensor cores: 128-token blocks with a ragged tail, and large logits (O rescale)
D64 = S.Workload("d64-bs128", 2, 3, 64, "bf16", (3, 10, 14), (2, 8, 8), 128, 0.85, 2, seed=17)
PEAKY_D64 = S.Workload("peaky-d64", 1, 3, 64, "bf16", (4, 16, 24), (1, 8, 16), 128, 0.97, 2,
                       seed=18, gen="gauss", peaky_head=2, peaky_scale=8.0)


# ----------------------------------------------------------------- permutation
@pytest.mark.parametrize("w", [S.WORKLOADS["tiny"], ODD, ODD128, S.WORKLOADS["wan1.3b-480p"]],
                         ids=lambda w: w.name)
def test_permute_bit_exact_and_inverse(w):
    q, _, _ = S.make_qkv(w, device="cuda")
    grid = F.Grid.make(w.grid, w.tile, w.block)
    perm = O.tile_order(*w.grid6)
    y = torch.full((w.B, w.H, grid.nb * w.block, w.d), 7.0, dtype=q.dtype, device="cuda")
    F.fvattn_permute(q, y, grid)
    ref = O.permute(_np(q), perm, w.block)
    assert np.array_equal(_np(y), ref)
    back = torch.empty_like(q)
    F.fvattn_permute(y, back, grid, inverse=True)
    assert torch.equal(back, q)


# ----------------------------------------------------------------- routing
@pytest.mark.parametrize("w", [S.WORKLOADS["tiny"], ODD, ODD128, SINGLE, TINY_BF16,
                               S.WORKLOADS["wan1.3b-480p"], S.WORKLOADS["wan14b-480p"]],
                         ids=lambda w: w.name)
def test_route_matches_oracle(w):
    q, k, _ = S.make_qkv(w, device="cuda")
    grid, qp, kp, kv_idx, kv_cnt, hw = _route_gpu(w, q, k)
    qn, kn = _np(q), _np(k)
    orc = O.route(qn, kn, w.grid6, w.block, w.p, w.k_min)
    assert np.array_equal(_np(qp), O.permute(qn, orc["perm"], w.block))
    assert np.array_equal(_np(kp), O.permute(kn, orc["perm"], w.block))
    idx, cnt = kv_idx.cpu().numpy(), kv_cnt.cpu().numpy()
    check_lists_valid(idx, cnt, grid.nb, w.k_min)
    assert np.array_equal(hw.cpu().numpy(), cnt.astype(np.int64).sum(-1))
    assert_mask_parity(compare_masks(mask_from_lists(idx, cnt, grid.nb), orc, w.p), w.name)


def test_route_p_one_and_large_floor_select_everything():
    w = ODD128.replace(p=1.0)
    q, k, _ = S.make_qkv(w, device="cuda")
    grid, _, _, kv_idx, kv_cnt, hw = _route_gpu(w, q, k)
    nb = grid.nb
    assert torch.all(kv_cnt == nb)
    assert torch.equal(kv_idx, torch.arange(nb, dtype=torch.int32, device="cuda").expand_as(kv_idx))
    w2 = ODD128.replace(p=0.3, k_min=1000)
    grid, _, _, kv_idx, kv_cnt, _ = _route_gpu(w2, q, k)
    assert torch.all(kv_cnt == nb)


def test_route_uniform_scores_tie_break():
    # q = 0 gives uniform importance: the cut takes the lowest block indices first.
    w = ODD128.replace(p=0.5, k_min=1)
    _, k, _ = S.make_qkv(w, device="cuda")
    q = torch.zeros_like(k)
    grid, _, _, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    nb = grid.nb
    orc_cnt = O.topp_topk_select(np.full(nb, 1.0 / nb), 0.5, 1)[1]
    c = kv_cnt.cpu().numpy()
    assert abs(int(c.min()) - orc_cnt) <= 1 and c.min() == c.max()
    first = kv_idx[..., : int(c.min())].cpu().numpy()
    assert np.array_equal(first, np.broadcast_to(np.arange(int(c.min())), first.shape))


# ----------------------------------------------------------------- attention
def _check_attention(w, q, k, v, op, mask, blocks, tol_max, tol_mean):
    # oracle inputs: the seeded q, k, v in the oracle's own tile order
    qpn, kpn, vpn = oracle_permuted(w, q, k, v)
    ref = O.masked_attention(qpn, kpn, vpn, mask, w.N, w.block, 1.0 / math.sqrt(w.d), blocks=blocks)
    got = _np(op)
    rows = np.zeros(ref.shape[:-1], dtype=bool)
    for (b, h, i) in blocks:
        rows[b, h, i * w.block:min((i + 1) * w.block, w.N)] = True
    mx, mean = attention_errors(got[rows], ref[rows])
    print(f"{w.name}: blocks={len(blocks)} max_abs={mx:.3e} mean_abs={mean:.3e}")
    assert np.all(np.isfinite(got[rows]))
    assert mx <= tol_max and mean <= tol_mean
    return mx, mean


def _sample_blocks(w, nb, cnt=None, per_head=6, seed=0):
    rng = np.random.default_rng(seed)
    out = []
    for b in range(w.B):
        for h in range(w.H):
            picks = set(rng.choice(nb, size=min(per_head, nb), replace=False).tolist())
            picks.add(nb - 1)                                   # the ragged tail block
            if cnt is not None:
                picks.add(int(np.argmax(cnt[b, h])))            # the head's heaviest row
            out += [(b, h, int(i)) for i in sorted(picks)]
    return out


@pytest.mark.parametrize("w", [S.WORKLOADS["tiny"], ODD, ODD128, SINGLE, TINY_BF16, PEAKY, BS64, BS64_ODD, D64,
                               PEAKY_D64],
                         ids=lambda w: w.name)
def test_sparse_and_dense_attention_all_blocks(w):
    q, k, v = S.make_qkv(w, device="cuda")
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    vp = torch.empty_like(qp)
    F.fvattn_permute(v, vp, grid)
    nb = grid.nb
    blocks = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(nb)]
    tol = (FP32_MAX_ABS, FP32_MAX_ABS) if w.dtype == "fp32" else (BF16_MAX_ABS, BF16_MEAN_ABS)
    op, _ = _attn_gpu(w, qp, kp, vp, kv_idx, kv_cnt)
    mask = mask_from_lists(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), nb)
    _check_attention(w, q, k, v, op, mask, blocks, *tol)
    opd, _ = _attn_gpu(w, qp, kp, vp)
    _check_attention(w, q, k, v, opd, np.ones_like(mask), blocks, *tol)


@pytest.mark.parametrize("name", ["wan1.3b-480p", "wan14b-480p"])
def test_tensor_core_attention_sampled(name):
    w = S.WORKLOADS[name]
    q, k, v = S.make_qkv(w, device="cuda")
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    vp = torch.empty_like(qp)
    F.fvattn_permute(v, vp, grid)
    nb = grid.nb
    cnt = kv_cnt.cpu().numpy()
    mask = mask_from_lists(kv_idx.cpu().numpy(), cnt, nb)
    blocks = _sample_blocks(w, nb, cnt, per_head=3)
    op, lse = _attn_gpu(w, qp, kp, vp, kv_idx, kv_cnt, lse=True)
    _check_attention(w, q, k, v, op, mask, blocks, BF16_MAX_ABS, BF16_MEAN_ABS)
    # lse of one row against the oracle's logits
    b, h, i = blocks[0]
    r = i * w.block
    cols = np.concatenate([np.arange(j * w.block, min((j + 1) * w.block, w.N)) for j in np.nonzero(mask[b, h, i])[0]])
    qo, ko = oracle_permuted(w, q, k)
    logits = (qo[b, h, r].astype(np.float64) @ ko[b, h, cols].astype(np.float64).T) / math.sqrt(w.d)
    ref_lse = logits.max() + math.log(np.exp(logits - logits.max()).sum())
    assert abs(float(lse[b, h, r]) - ref_lse) < 1e-3
    opd, _ = _attn_gpu(w, qp, kp, vp)
    _check_attention(w, q, k, v, opd, np.ones_like(mask), blocks[: 4 * w.H: 4],
                     BF16_MAX_ABS, BF16_MEAN_ABS)


@pytest.mark.parametrize("w", [ODD128, D64], ids=lambda w: w.name)
def test_sparse_with_full_lists_is_bitwise_dense(w):
    q, k, v = S.make_qkv(w, device="cuda")
    grid = F.Grid.make(w.grid, w.tile, w.block)
    nb = grid.nb
    qp = torch.empty((w.B, w.H, nb * w.block, w.d), dtype=q.dtype, device="cuda")
    kp, vp = torch.empty_like(qp), torch.empty_like(qp)
    for x, y in ((q, qp), (k, kp), (v, vp)):
        F.fvattn_permute(x, y, grid)
    kv_idx = torch.arange(nb, dtype=torch.int32, device="cuda").expand(w.B, w.H, nb, nb).contiguous()
    kv_cnt = torch.full((w.B, w.H, nb), nb, dtype=torch.int32, device="cuda")
    a, _ = _attn_gpu(w, qp, kp, vp, kv_idx, kv_cnt)
    b, _ = _attn_gpu(w, qp, kp, vp)
    assert torch.equal(a, b)


def test_list_order_does_not_matter_beyond_rounding():
    w = ODD128
    q, k, v = S.make_qkv(w, device="cuda")
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    vp = torch.empty_like(qp)
    F.fvattn_permute(v, vp, grid)
    a, _ = _attn_gpu(w, qp, kp, vp, kv_idx, kv_cnt)
    rev = kv_idx.clone()
    for row in np.ndindex(*kv_cnt.shape):
        c = int(kv_cnt[row])
        rev[row][:c] = torch.flip(kv_idx[row][:c], dims=[0])
    b, _ = _attn_gpu(w, qp, kp, vp, rev, kv_cnt)
    npad_rows = torch.arange(qp.shape[2], device="cuda") < w.N
    d = (a.float() - b.float()).abs()[:, :, npad_rows]
    assert float(d.max()) <= 2e-2


def test_full_path_720p_sampled():
    """The bench workload end to end through FVAttnPath, every mask row, sampled outputs."""
    w = S.WORKLOADS["wan14b-720p"]
    q, k, v = S.make_qkv(w, device="cuda")
    path = F.FVAttnPath(w.B, w.H, w.grid, w.tile, w.block, w.d, torch.bfloat16, w.p, w.k_min)
    out = path(q, k, v)
    torch.cuda.synchronize()
    assert F.fvattn_workspace_status(path.ws_route) == F.FVATTN_OK
    assert F.fvattn_workspace_status(path.ws_attn) == F.FVATTN_OK
    nb = path.nb
    idx, cnt = path.kv_idx.cpu().numpy(), path.kv_cnt.cpu().numpy()
    check_lists_valid(idx, cnt, nb, w.k_min)
    qn, kn = _np(q), _np(k)
    orc = O.route(qn, kn, w.grid6, w.block, w.p, w.k_min)
    mask = mask_from_lists(idx, cnt, nb)
    assert_mask_parity(compare_masks(mask, orc, w.p), f"720p density={cnt.mean() / nb:.3f}")
    assert np.array_equal(path.head_work.cpu().numpy(), cnt.astype(np.int64).sum(-1))
    # sampled output rows in ORIGINAL order against the oracle on the GPU's mask,
    # one head at a time to bound host memory
    perm = orc["perm"]
    blocks = _sample_blocks(w, nb, cnt, per_head=1, seed=3)
    vn = _np(v)
    got = _np(out)
    scale = 1.0 / math.sqrt(w.d)
    errs_max, errs_sum, n = 0.0, 0.0, 0
    for (b, h) in sorted({(b, h) for (b, h, _) in blocks}):
        qp, kp, vp = (O.permute(x[b, h].astype(np.float64), perm, w.block) for x in (qn, kn, vn))
        for (bb, hh, i) in blocks:
            if (bb, hh) != (b, h):
                continue
            ref = O.masked_attention_rows(qp, kp, vp, mask[b, h, i], w.N, w.block, scale, i)
            pos = np.arange(i * w.block, i * w.block + ref.shape[0])
            e = np.abs(got[b, h, perm[pos]] - ref)
            errs_max = max(errs_max, float(e.max()))
            errs_sum += float(e.sum())
            n += e.size
    print(f"720p outputs: blocks={len(blocks)} max_abs={errs_max:.3e} mean_abs={errs_sum / n:.3e}")
    assert errs_max <= BF16_MAX_ABS and errs_sum / n <= BF16_MEAN_ABS


def test_batch_of_two_tensor_core():
    w = S.WORKLOADS["wan1.3b-480p"].replace(name="b2-480p-h4", B=2, H=4)
    q, k, v = S.make_qkv(w, device="cuda")
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    vp = torch.empty_like(qp)
    F.fvattn_permute(v, vp, grid)
    nb = grid.nb
    cnt = kv_cnt.cpu().numpy()
    mask = mask_from_lists(kv_idx.cpu().numpy(), cnt, nb)
    op, _ = _attn_gpu(w, qp, kp, vp, kv_idx, kv_cnt)
    _check_attention(w, q, k, v, op, mask, _sample_blocks(w, nb, cnt, per_head=4),
                     BF16_MAX_ABS, BF16_MEAN_ABS)


def test_route_720p_bs64_sampled_heads():
    """64-token blocks (1x8x8 tiles) at the 720p shape: every query block of 8 heads against
    the oracle's routing (the rest of the heads are routed by the same launch)."""
    w = S.WORKLOADS["wan14b-720p"].replace(name="wan14b-720p-bs64", block=64, tile=(1, 8, 8))
    q, k, _ = S.make_qkv(w, device="cuda")
    grid, qp, kp, kv_idx, kv_cnt, hw = _route_gpu(w, q, k)
    heads = list(range(0, w.H, 5))
    orc = O.route(_np(q[:, heads]), _np(k[:, heads]), w.grid6, w.block, w.p, w.k_min)
    idx, cnt = kv_idx[:, heads].cpu().numpy(), kv_cnt[:, heads].cpu().numpy()
    check_lists_valid(idx, cnt, grid.nb, w.k_min)
    assert np.array_equal(hw.cpu().numpy(), kv_cnt.cpu().numpy().astype(np.int64).sum(-1))
    assert_mask_parity(compare_masks(mask_from_lists(idx, cnt, grid.nb), orc, w.p), w.name)


@pytest.mark.parametrize("w", [ODD128, S.WORKLOADS["wan1.3b-480p"], BS64], ids=lambda w: w.name)
def test_lists_in_importance_order(w):
    """The same sets as the routed lists, reordered by descending score: against the
    oracle's scores every list is non-increasing up to the near-cut tolerance, and the
    attention result does not change beyond rounding."""
    q, k, v = S.make_qkv(w, device="cuda")
    grid = F.Grid.make(w.grid, w.tile, w.block)
    nb, npad = grid.nb, grid.nb * w.block
    dev = q.device
    qp = torch.empty((w.B, w.H, npad, w.d), dtype=q.dtype, device=dev)
    kp = torch.empty_like(qp)
    kv_idx = torch.empty((w.B, w.H, nb, nb), dtype=torch.int32, device=dev)
    kv_cnt = torch.empty((w.B, w.H, nb), dtype=torch.int32, device=dev)
    hw = torch.empty((w.B, w.H), dtype=torch.int64, device=dev)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_route(q, k, grid, w.p, w.k_min, kv_idx, kv_cnt, hw, ws, qp_out=qp, kp_out=kp)
    asc = kv_idx.clone()
    F.fvattn_order_lists_by_importance(kv_idx, kv_cnt, w.N, w.d, w.block, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    orc = O.route(_np(q), _np(k), w.grid6, w.block, w.p, w.k_min)
    idx, cnt, idx_asc = kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), asc.cpu().numpy()
    for row in np.ndindex(*cnt.shape):
        c = int(cnt[row])
        got = idx[row][:c]
        assert np.array_equal(np.sort(got), idx_asc[row][:c]), row
        # the GPU orders by its fp32 logits; scores closer than their rounding may swap
        s = orc["scores"][row][got]
        assert np.all(s[1:] <= s[:-1] * (1 + 1e-4)), (row, s[:8])
    vp = torch.empty_like(qp)
    F.fvattn_permute(v, vp, grid)
    a, _ = _attn_gpu(w, qp, kp, vp, asc, kv_cnt)
    b, _ = _attn_gpu(w, qp, kp, vp, kv_idx, kv_cnt)
    d = (a.float() - b.float()).abs()[:, :, : w.N]
    assert float(d.max()) <= 2e-2


def test_importance_order_breaks_ties_by_block_index():
    # q = 0: every score of a row is equal, so the order is ascending block index
    w = ODD128.replace(p=0.5, k_min=1)
    _, k, _ = S.make_qkv(w, device="cuda")
    q = torch.zeros_like(k)
    grid = F.Grid.make(w.grid, w.tile, w.block)
    nb = grid.nb
    kv_idx = torch.empty((w.B, w.H, nb, nb), dtype=torch.int32, device="cuda")
    kv_cnt = torch.empty((w.B, w.H, nb), dtype=torch.int32, device="cuda")
    hw = torch.empty((w.B, w.H), dtype=torch.int64, device="cuda")
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, w.B, w.H, w.N, w.d, w.block), "cuda")
    F.fvattn_route(q, k, grid, w.p, w.k_min, kv_idx, kv_cnt, hw, ws)
    asc = kv_idx.clone()
    F.fvattn_order_lists_by_importance(kv_idx, kv_cnt, w.N, w.d, w.block, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    c = int(kv_cnt.min())
    assert torch.equal(kv_idx[..., :c], asc[..., :c])
