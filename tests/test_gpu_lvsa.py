"""GPU parity of the LVSA static mask generator (fvattn_lvsa_lists) against the
oracle: lists, counts and per-head work bit for bit; then block-sparse attention
over LVSA lists against the oracle's masked attention."""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from oracle import lvsa_oracle as L
from parity import BF16_MAX_ABS, BF16_MEAN_ABS, attention_errors, mask_from_lists

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_video_b200 as F


def _lvsa_gpu(grid_t, tile, bs, W, Tper, step, B=1, H=3):
    grid = F.Grid.make(grid_t, tile, bs)
    nb = grid.nb
    dev = torch.device("cuda")
    kv_idx = torch.full((B, H, nb, nb), -3, dtype=torch.int32, device=dev)
    kv_cnt = torch.empty((B, H, nb), dtype=torch.int32, device=dev)
    hw = torch.empty((B, H), dtype=torch.int64, device=dev)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_LVSA, B, H, grid.N, 64, bs), dev)
    F.fvattn_lvsa_lists(grid, W, Tper, step, kv_idx, kv_cnt, hw, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    return grid, kv_idx, kv_cnt, hw


CASES = [
    ((9, 10, 14), (2, 8, 8), 128, 1, 3, 2),      # ragged tiles, blocks straddle tiles
    ((13, 12, 20), (1, 8, 8), 64, 0, 4, 3),      # bs 64, window 0
    ((40, 8, 8), (1, 8, 8), 64, 3, 6, 7),        # one frame per block; 2-word frame masks
    ((100, 4, 4), (1, 4, 4), 64, 2, 9, 11),      # 4 frames per block; 4-word frame masks
    ((5, 9, 7), (3, 2, 3), 64, 4, 2, 0),         # window wider than the video: dense
    ((21, 30, 52), (2, 8, 8), 128, 2, 8, 0),     # 480p shape
    ((21, 45, 80), (2, 8, 8), 128, 2, 8, 5),     # 720p shape
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[0])) + f"-bs{c[2]}-W{c[3]}-P{c[4]}-s{c[5]}")
def test_lvsa_lists_match_oracle(case):
    grid_t, tile, bs, W, Tper, step = case
    grid, kv_idx, kv_cnt, hw = _lvsa_gpu(grid_t, tile, bs, W, Tper, step)
    perm = O.tile_order(*grid_t, *tile)
    want = L.lvsa_block_mask(perm, grid_t, bs, W, Tper, step)
    idx, cnt = kv_idx.cpu().numpy(), kv_cnt.cpu().numpy()
    nb = grid.nb
    for h in range(cnt.shape[1]):
        assert np.array_equal(cnt[0, h], want.sum(-1)), h
        for i in range(nb):
            assert np.array_equal(idx[0, h, i, :cnt[0, h, i]], np.nonzero(want[i])[0]), (h, i)
            assert np.all(idx[0, h, i, cnt[0, h, i]:] == -3)      # entries past cnt untouched
    assert np.array_equal(hw.cpu().numpy(), np.full(hw.shape, want.sum()))
    print(f"{case}: nb={nb} density {want.mean():.3f}")


def test_frame_aligned_lists_equal_the_frame_pattern():
    grid, kv_idx, kv_cnt, _ = _lvsa_gpu((40, 8, 8), (1, 8, 8), 64, 3, 6, 7, H=1)
    mask = mask_from_lists(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), grid.nb)[0, 0]
    assert np.array_equal(mask, L.frame_mask(40, 3, 6, 7))
    # every query frame attends the same number of frames
    assert len(set(mask.sum(-1).tolist())) == 1


def test_sparse_attention_over_lvsa_lists():
    w = S.Workload("lvsa-attn", 1, 2, 128, "bf16", (8, 16, 24), (2, 8, 8), 128, 0.9, 1, seed=21)
    q, k, v = S.make_qkv(w, device="cuda")
    grid, kv_idx, kv_cnt, _ = _lvsa_gpu(w.grid, w.tile, w.block, 0, 8, 1, B=w.B, H=w.H)   # density 0.5
    qp, kp, vp = (torch.empty((w.B, w.H, grid.nb * w.block, w.d), dtype=q.dtype, device="cuda")
                  for _ in range(3))
    for x, y in ((q, qp), (k, kp), (v, vp)):
        F.fvattn_permute(x, y, grid)
    op = torch.empty_like(qp)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_SPARSE_FWD, w.B, w.H, w.N, w.d, w.block), "cuda")
    F.fvattn_sparse_fwd(qp, kp, vp, op, kv_idx, kv_cnt, w.N, w.block, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    perm = O.tile_order(*w.grid, *w.tile)
    want = L.lvsa_block_mask(perm, w.grid, w.block, 0, 8, 1)       # the oracle's mask
    mask = mask_from_lists(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), grid.nb)
    assert all(np.array_equal(mask[0, h], want) for h in range(w.H))
    assert 0.2 < want.mean() < 0.9
    to_np = lambda t: t.float().cpu().numpy()
    ref = O.masked_attention(*(O.permute(to_np(x), perm, w.block) for x in (q, k, v)),
                             np.broadcast_to(want, mask.shape), w.N, w.block, 1.0 / math.sqrt(w.d))
    mx, mean = attention_errors(to_np(op)[:, :, :w.N], ref[:, :, :w.N])
    assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, (mx, mean)
    print(f"lvsa attention: density {mask.mean():.3f} max_abs {mx:.2e} mean_abs {mean:.2e}")
