"""GPU: invalid KV lists are turned into an error status by the kernels' own
bounds checks (a count outside [1, nb] is clamped, a block index outside [0, nb)
is dropped or clamped), and every kernel still runs to completion, so the call
returns and the status word reads FVATTN_ERR_INVALID_ARG. Rows with valid lists
keep their exact results."""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import BF16_MAX_ABS, FP32_MAX_ABS, attention_errors, mask_from_lists

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_video_b200 as F


def _lists(w, nb, dev):
    # every query block attends itself and block 0 (ascending), then two rows are broken
    idx = torch.zeros((w.B, w.H, nb, nb), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.H, nb), dtype=torch.int32, device=dev)
    for i in range(nb):
        lst = sorted({0, i})
        idx[..., i, :len(lst)] = torch.tensor(lst, dtype=torch.int32, device=dev)
        cnt[..., i] = len(lst)
    return idx, cnt


@pytest.mark.parametrize("w", [
    S.Workload("err-bf16", 1, 2, 128, "bf16", (4, 16, 16), (1, 8, 16), 128, 0.9, 1, seed=61),
    S.Workload("err-bf16-bs64", 1, 2, 128, "bf16", (5, 12, 20), (1, 8, 8), 64, 0.9, 1, seed=62),
    S.Workload("err-fp32", 1, 2, 64, "fp32", (4, 8, 8), (1, 8, 8), 64, 0.9, 1, seed=63),
], ids=lambda w: w.name)
def test_invalid_lists_are_reported_and_valid_rows_kept(w):
    dev = torch.device("cuda")
    q, k, v = S.make_qkv(w, device=dev)
    grid = F.Grid.make(w.grid, w.tile, w.block)
    nb = grid.nb
    qp, kp, vp = (torch.empty((w.B, w.H, nb * w.block, w.d), dtype=q.dtype, device=dev) for _ in range(3))
    for x, y in ((q, qp), (k, kp), (v, vp)):
        F.fvattn_permute(x, y, grid)
    idx, cnt = _lists(w, nb, dev)
    good_idx, good_cnt = idx.clone(), cnt.clone()
    cnt[0, 0, 1] = 0                 # count below 1
    idx[0, 1, 2, 1] = nb + 5         # block index past the end
    cnt[0, 1, 3] = nb + 9            # count above nb
    op = torch.zeros_like(qp)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_SPARSE_FWD, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_sparse_fwd(qp, kp, vp, op, idx, cnt, w.N, w.block, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_ERR_INVALID_ARG
    # the broken rows' neighbours in other query blocks are untouched by the clamping
    mask = mask_from_lists(good_idx.cpu().numpy(), good_cnt.cpu().numpy(), nb)
    to_np = lambda t: t.float().cpu().numpy()
    perm = O.tile_order(*w.grid, *w.tile)      # the oracle's own permutation of the seeded inputs
    ref = O.masked_attention(*(O.permute(to_np(x), perm, w.block) for x in (q, k, v)), mask, w.N, w.block,
                             1.0 / math.sqrt(w.d))
    bs = w.block
    for (b, h, i) in [(0, 0, 0), (0, 1, 0), (0, 0, nb - 1)]:
        rows = slice(i * bs, min((i + 1) * bs, w.N))
        mx, _ = attention_errors(to_np(op)[b, h, rows], ref[b, h, rows])
        assert mx <= (FP32_MAX_ABS if w.dtype == "fp32" else BF16_MAX_ABS), (b, h, i, mx)
    # a clean call on the same workspace reports OK again
    F.fvattn_sparse_fwd(qp, kp, vp, op, good_idx, good_cnt, w.N, w.block, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK


def test_invalid_lists_in_the_importance_kernels_are_reported():
    w = S.Workload("err-imp", 1, 2, 64, "fp32", (4, 8, 8), (1, 8, 8), 64, 0.9, 1, seed=64)
    dev = torch.device("cuda")
    nb = O.num_blocks(w.N, w.block)
    npad = nb * w.block
    blse = torch.zeros((w.B, w.H, nb, npad), dtype=torch.float32, device=dev)
    lse = torch.zeros((w.B, w.H, npad), dtype=torch.float32, device=dev)
    imp = torch.empty((w.B, w.H, nb, nb), dtype=torch.float32, device=dev)
    rec = torch.empty((w.B, w.H, nb), dtype=torch.float32, device=dev)
    idx, cnt = _lists(w, nb, dev)
    idx[0, 0, 1, 0] = -4
    cnt[0, 1, 2] = 0
    wsd = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_DIAG, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_block_importance(blse, lse, imp, w.N, w.block, wsd, kv_idx=idx, kv_cnt=cnt)
    assert F.fvattn_workspace_status(wsd) == F.FVATTN_ERR_INVALID_ARG
    F.fvattn_attention_recall(imp, idx, cnt, rec, w.N, w.block, wsd)
    assert F.fvattn_workspace_status(wsd) == F.FVATTN_ERR_INVALID_ARG
    assert torch.isfinite(imp).all() and torch.isfinite(rec).all()


def test_invalid_lists_in_the_fp8v_path_are_reported():
    w = S.Workload("err-fp8v", 1, 2, 128, "bf16", (5, 12, 20), (1, 8, 8), 64, 0.9, 1, seed=65)
    dev = torch.device("cuda")
    q, k, v = S.make_qkv(w, device=dev)
    grid = F.Grid.make(w.grid, w.tile, w.block)
    nb = grid.nb
    qp, kp, vp = (torch.empty((w.B, w.H, nb * w.block, w.d), dtype=q.dtype, device=dev) for _ in range(3))
    for x, y in ((q, qp), (k, kp), (v, vp)):
        F.fvattn_permute(x, y, grid)
    vq = torch.empty(vp.shape, dtype=torch.uint8, device=dev)
    vs = torch.empty((w.B, w.H, w.d), dtype=torch.float32, device=dev)
    wsq = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_QUANT_V, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_quantize_v(vp, vq, vs, w.N, w.block, wsq)
    assert F.fvattn_workspace_status(wsq) == F.FVATTN_OK
    idx, cnt = _lists(w, nb, dev)
    good_idx, good_cnt = idx.clone(), cnt.clone()
    cnt[0, 0, 1] = 0
    idx[0, 1, 2, 1] = -3
    op = torch.zeros_like(qp)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_SPARSE_FWD, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_sparse_fwd_fp8v(qp, kp, vq, vs, op, idx, cnt, w.N, w.block, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_ERR_INVALID_ARG
    assert torch.isfinite(op[:, :, : w.N]).all()
    # rows of untouched query blocks match a clean call up to rounding order (a broken
    # list in the same 256-row unit changes how the unit's entries pair into steps)
    op_good = torch.zeros_like(qp)
    F.fvattn_sparse_fwd_fp8v(qp, kp, vq, vs, op_good, good_idx, good_cnt, w.N, w.block, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    bs = w.block
    for (b, h, i) in [(0, 0, 0), (0, 1, 0), (0, 0, nb - 1)]:
        rows = slice(i * bs, min((i + 1) * bs, w.N))
        mx, _ = attention_errors(op[b, h, rows].float().cpu().numpy(), op_good[b, h, rows].float().cpu().numpy())
        assert mx <= BF16_MAX_ABS, (b, h, i, mx)


def test_bounded_waits_run_out_and_report_a_timeout():
    """The waits every kernel uses, on barriers nothing arrives at: each gives up after
    the limit, the abort flag releases the second waiter, the status word reads
    FVATTN_ERR_TIMEOUT, and the context keeps working (no fault, no hang)."""
    dev = torch.device("cuda")
    res = torch.full((8,), -1, dtype=torch.int64, device=dev)
    ws = F.alloc_workspace(256, dev)
    F.fvattn_wait_selftest(res, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_ERR_TIMEOUT
    r = res.cpu().tolist()
    limit = r[6]
    assert limit == 2_000_000_000
    assert r[0] == 0 and limit <= r[1] < limit + 500_000_000, r          # ran out at the limit
    assert r[2] == 0 and r[3] < limit + 500_000_000, r                   # released, not stuck
    assert r[4] == 0 and limit <= r[5] < limit + 500_000_000, r          # drain wait bounded too
    assert r[7] == 1, r                                                  # abort flag raised
    # the same workspace and context still run a kernel and report OK
    w = S.Workload("after-timeout", 1, 2, 128, "bf16", (2, 8, 16), (1, 8, 16), 128, 0.9, 1, seed=66)
    q, k, v = S.make_qkv(w, device=dev)
    grid = F.Grid.make(w.grid, w.tile, w.block)
    qp, kp, vp = (torch.empty((w.B, w.H, grid.nb * w.block, w.d), dtype=q.dtype, device=dev) for _ in range(3))
    for x, y in ((q, qp), (k, kp), (v, vp)):
        F.fvattn_permute(x, y, grid)
    op = torch.empty_like(qp)
    F.fvattn_dense_fwd(qp, kp, vp, op, w.N, w.block, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    assert torch.isfinite(op[:, :, : w.N].float()).all()
