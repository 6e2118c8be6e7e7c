"""GPU edge cases through the C-ABI against the oracle: degenerate grids (one
token, one row of tokens, a single partial block), and the largest block count
the router supports (about 4,000 key blocks of 64 tokens), at which the route is
checked on every row and attention on sampled query blocks."""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import (BF16_MAX_ABS, BF16_MEAN_ABS, FP32_MAX_ABS, assert_mask_parity, attention_errors,
                    check_lists_valid, compare_masks, mask_from_lists)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_video_b200 as F


def _np(t):
    return t.detach().float().cpu().numpy()


def _full_path(w, order="tiles"):
    q, k, v = S.make_qkv(w, device="cuda")
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    path = F.FVAttnPath(w.B, w.H, w.grid, w.tile, w.block, w.d, dt, w.p, w.k_min, order=order)
    out = _np(path(q, k, v))
    assert F.fvattn_workspace_status(path.ws_route) == F.FVATTN_OK
    assert F.fvattn_workspace_status(path.ws_attn) == F.FVATTN_OK
    return q, k, v, path, out


@pytest.mark.parametrize("w", [
    S.Workload("one-token", 1, 2, 64, "fp32", (1, 1, 1), (1, 1, 1), 64, 0.9, 1, seed=51),
    S.Workload("one-token-bf16", 1, 2, 128, "bf16", (1, 1, 1), (1, 8, 8), 128, 0.9, 1, seed=52),
    S.Workload("one-row", 1, 1, 128, "bf16", (1, 1, 77), (1, 1, 8), 64, 0.5, 1, seed=53),
    S.Workload("partial-block", 2, 2, 128, "bf16", (3, 5, 7), (2, 2, 2), 128, 0.9, 1, seed=54),
], ids=lambda w: w.name)
def test_degenerate_grids(w):
    q, k, v, path, out = _full_path(w)
    qn, kn, vn = _np(q), _np(k), _np(v)
    orc = O.route(qn, kn, w.grid6, w.block, w.p, w.k_min)
    idx, cnt = path.kv_idx.cpu().numpy(), path.kv_cnt.cpu().numpy()
    check_lists_valid(idx, cnt, path.nb, w.k_min)
    assert_mask_parity(compare_masks(mask_from_lists(idx, cnt, path.nb), orc, w.p), w.name)
    mask = mask_from_lists(idx, cnt, path.nb)
    ref = O.masked_attention(*(O.permute(x, orc["perm"], w.block) for x in (qn, kn, vn)), mask, w.N,
                             w.block, 1.0 / math.sqrt(w.d))
    ref = O.inverse_permute(ref, orc["perm"])
    mx, mean = attention_errors(out, ref)
    if w.dtype == "fp32":
        assert mx <= FP32_MAX_ABS, mx
    else:
        assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, (mx, mean)
    if w.N == 1:
        # a single key: the output is that token's V row
        assert np.allclose(out, vn, atol=1e-2 if w.dtype == "bf16" else 1e-6)


def test_largest_supported_block_count():
    # 21 x 80 x 152 tokens = 255,360 -> 3,990 blocks of 64 (the router holds about 4,000)
    w = S.Workload("max-blocks", 1, 1, 128, "bf16", (21, 80, 152), (1, 8, 8), 64, 0.9, 4, seed=55)
    assert O.num_blocks(w.N, w.block) == 3990
    q, k, v, path, out = _full_path(w)
    qn, kn, vn = _np(q), _np(k), _np(v)
    orc = O.route(qn, kn, w.grid6, w.block, w.p, w.k_min)
    idx, cnt = path.kv_idx.cpu().numpy(), path.kv_cnt.cpu().numpy()
    check_lists_valid(idx, cnt, path.nb, w.k_min)
    mask = mask_from_lists(idx, cnt, path.nb)
    mres = compare_masks(mask, orc, w.p)
    assert_mask_parity(mres, w.name)
    perm = orc["perm"]
    qp, kp, vp = (O.permute(x[0, 0], perm, w.block) for x in (qn, kn, vn))
    outp = O.permute(out[0, 0], perm, w.block)
    rng = np.random.default_rng(3)
    for i in list(rng.integers(0, path.nb, 6)) + [path.nb - 1]:
        ref = O.masked_attention_rows(qp, kp, vp, mask[0, 0, i], w.N, w.block, 1.0 / math.sqrt(w.d), int(i))
        got = outp[i * w.block:i * w.block + ref.shape[0]]
        mx, mean = attention_errors(got, ref)
        assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, (i, mx, mean)
    print(f"max-blocks: nb={path.nb} density {mask.mean():.3f} mismatched={mres['mismatched']} "
          f"borderline={mres['borderline']}")


def test_binding_rejects_mismatched_buffers_before_any_launch():
    """The binding checks every buffer's shape, dtype and device against the call (the
    library itself sees only pointers)."""
    w = S.Workload("bind", 1, 2, 128, "bf16", (2, 8, 15), (1, 8, 16), 128, 0.9, 1, seed=67)   # N=240, ragged
    dev = torch.device("cuda")
    q, k, v = S.make_qkv(w, device=dev)
    grid = F.Grid.make(w.grid, w.tile, w.block)
    nb, npad = grid.nb, grid.nb * w.block
    idx = torch.empty((1, 2, nb, nb), dtype=torch.int32, device=dev)
    cnt = torch.empty((1, 2, nb), dtype=torch.int32, device=dev)
    hw = torch.empty((1, 2), dtype=torch.int64, device=dev)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, 1, 2, w.N, w.d, w.block), dev)
    with pytest.raises(ValueError):      # list buffer one row short
        F.fvattn_route(q, k, grid, 0.9, 1, idx[:, :, :, :-1].contiguous(), cnt, hw, ws)
    with pytest.raises(TypeError):       # k in another dtype than q
        F.fvattn_route(q, k.float(), grid, 0.9, 1, idx, cnt, hw, ws)
    with pytest.raises(TypeError):       # counts in int64
        F.fvattn_route(q, k, grid, 0.9, 1, idx, cnt.long(), hw, ws)
    with pytest.raises(ValueError):      # permuted output without the pad rows
        F.fvattn_route(q, k, grid, 0.9, 1, idx, cnt, hw, ws, qp_out=torch.empty_like(q))
    qp = torch.zeros((1, 2, npad, w.d), dtype=q.dtype, device=dev)
    wsa = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_SPARSE_FWD, 1, 2, w.N, w.d, w.block), dev)
    with pytest.raises(ValueError):      # output of the wrong length
        F.fvattn_sparse_fwd(qp, qp, qp, torch.empty_like(q), idx, cnt, w.N, w.block, wsa)
    with pytest.raises(ValueError):      # lse of the wrong length
        F.fvattn_dense_fwd(qp, qp, qp, torch.empty_like(qp), w.N, w.block, wsa,
                           lse=torch.empty((1, 2, w.N), dtype=torch.float32, device=dev))
    with pytest.raises(ValueError):      # x of the wrong length for the grid
        F.fvattn_permute(qp, torch.empty_like(qp), grid)
    # the well-formed calls go through
    F.fvattn_route(q, k, grid, 0.9, 1, idx, cnt, hw, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
