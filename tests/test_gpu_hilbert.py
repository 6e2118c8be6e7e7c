"""GPU parity of the Hilbert block order (FVATTN_ORDER_TABLE grids with the table
from fvattn_hilbert_table) against the oracle: the table and every permutation
bit for bit, routing masks under the borderline rule, LVSA lists bit for bit, and
the whole path's output in original order within the bf16 gate."""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from oracle import hilbert_oracle as Hb
from oracle import lvsa_oracle as L
from parity import (BF16_MAX_ABS, BF16_MEAN_ABS, assert_mask_parity, attention_errors, check_lists_valid,
                    compare_masks, mask_from_lists)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_video_b200 as F


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


@pytest.mark.parametrize("thw", [(1, 1, 1), (3, 5, 7), (2, 8, 8), (7, 1, 13), (21, 30, 52), (21, 45, 80)],
                         ids=lambda g: "x".join(map(str, g)))
def test_hilbert_table_matches_oracle(thw):
    table = F.fvattn_hilbert_table(thw, 128)
    want = Hb.hilbert_order(*thw)
    assert np.array_equal(table.cpu().numpy(), want)


HW = S.Workload("hilbert-bf16", 1, 3, 128, "bf16", (5, 12, 20), (1, 8, 8), 128, 0.9, 2, seed=31)
HW64 = S.Workload("hilbert-fp32-bs64", 2, 2, 64, "fp32", (6, 10, 9), (1, 8, 8), 64, 0.8, 1, seed=32)


@pytest.mark.parametrize("w", [HW, HW64], ids=lambda w: w.name)
def test_permute_and_route_in_hilbert_order(w):
    q, k, v = S.make_qkv(w, device="cuda")
    table = F.fvattn_hilbert_table(w.grid, w.block)
    grid = F.Grid.make(w.grid, w.tile, w.block, table=table)
    perm = Hb.hilbert_order(*w.grid)
    y = torch.full((w.B, w.H, grid.nb * w.block, w.d), 5.0, dtype=v.dtype, device="cuda")
    F.fvattn_permute(v, y, grid)
    assert np.array_equal(_np(y), O.permute(_np(v), perm, w.block))
    back = torch.empty_like(v)
    F.fvattn_permute(y, back, grid, inverse=True)
    assert torch.equal(back, v)
    # routing over Hilbert-ordered blocks
    nb = grid.nb
    qp, kp = torch.empty_like(y), torch.empty_like(y)
    kv_idx = torch.empty((w.B, w.H, nb, nb), dtype=torch.int32, device="cuda")
    kv_cnt = torch.empty((w.B, w.H, nb), dtype=torch.int32, device="cuda")
    hw = torch.empty((w.B, w.H), dtype=torch.int64, device="cuda")
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, w.B, w.H, w.N, w.d, w.block), "cuda")
    F.fvattn_route(q, k, grid, w.p, w.k_min, kv_idx, kv_cnt, hw, ws, qp_out=qp, kp_out=kp)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    qn, kn = _np(q), _np(k)
    orc = O.route(qn, kn, w.grid6, w.block, w.p, w.k_min, perm=perm)
    assert np.array_equal(_np(qp), O.permute(qn, perm, w.block))
    idx, cnt = kv_idx.cpu().numpy(), kv_cnt.cpu().numpy()
    check_lists_valid(idx, cnt, nb, w.k_min)
    assert_mask_parity(compare_masks(mask_from_lists(idx, cnt, nb), orc, w.p), w.name)


def test_lvsa_lists_in_hilbert_order():
    thw, bs = (12, 8, 16), 64
    table = F.fvattn_hilbert_table(thw, bs)
    grid = F.Grid.make(thw, (1, 1, 1), bs, table=table)
    nb = grid.nb
    kv_idx = torch.empty((1, 2, nb, nb), dtype=torch.int32, device="cuda")
    kv_cnt = torch.empty((1, 2, nb), dtype=torch.int32, device="cuda")
    hw = torch.empty((1, 2), dtype=torch.int64, device="cuda")
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_LVSA, 1, 2, grid.N, 64, bs), "cuda")
    F.fvattn_lvsa_lists(grid, 1, 4, 2, kv_idx, kv_cnt, hw, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    want = L.lvsa_block_mask(Hb.hilbert_order(*thw), thw, bs, 1, 4, 2)
    got = mask_from_lists(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), nb)
    assert np.array_equal(got[0, 0], want) and np.array_equal(got[0, 1], want)


def test_full_path_in_hilbert_order():
    w = HW
    q, k, v = S.make_qkv(w, device="cuda")
    path = F.FVAttnPath(w.B, w.H, w.grid, w.tile, w.block, w.d, torch.bfloat16, w.p, w.k_min, order="hilbert")
    out = _np(path(q, k, v))
    assert F.fvattn_workspace_status(path.ws_attn) == F.FVATTN_OK
    perm = Hb.hilbert_order(*w.grid)
    qn, kn, vn = _np(q), _np(k), _np(v)
    mask = mask_from_lists(path.kv_idx.cpu().numpy(), path.kv_cnt.cpu().numpy(), path.nb)
    ref = O.masked_attention(*(O.permute(x, perm, w.block) for x in (qn, kn, vn)), mask, w.N, w.block,
                             1.0 / math.sqrt(w.d))
    ref = O.inverse_permute(ref, perm)
    mx, mean = attention_errors(out, ref)
    assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, (mx, mean)
    print(f"hilbert path: density {mask.mean():.3f} max_abs {mx:.2e} mean_abs {mean:.2e}")
