"""GPU: online softmax when a row's max jumps far above its running max [GSRS §A.1: earlier
partial results are rescaled when the max grows], against the oracle's masked attention
and row log-sum-exp on the oracle's own permutation of the same inputs.

The tensor-core kernel raises a row's running max, and rescales O in TMEM, when a step's
max exceeds it by more than 8 in base 2; the decision is per row, the O load and store
are taken by the whole warp. Here a third of the query tokens carry a large component
along one channel, and two keys, placed in later key blocks of every list, carry a larger
one: their logits lie about 76 and 153 (in base 2) above everything else, so those rows
rescale twice and the other rows of the same warps do not. One planted key sits in the
first 64 keys of its 128-key step and one in the second 64. The same inputs run dense,
where every key block is a step."""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import BF16_MAX_ABS, BF16_MEAN_ABS, attention_errors

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_video_b200 as F

LIST = [0, 5, 9, 13, 20, 30]      # every row's key blocks (ascending)


def _planted(w, block):
    """Seeded q, k, v (host, bf16) with the large components; the planted key positions
    are given in the oracle's tile order and mapped back to token indices."""
    q, k, v = S.make_qkv(w)
    perm = O.tile_order(*w.grid, *w.tile)
    q = q.float()
    k = k.float()
    q[:, :, 0::3, 0] = 4.0
    # (key block, column within the block, value): 4 x 150 / sqrt(128) x log2(e) = 76.5,
    # 4 x 300 / sqrt(128) x log2(e) = 153
    first = (9, 10, 150.0)
    second = (30, 100, 300.0) if block == 128 else (30, 40, 300.0)
    for b, c, val in (first, second):
        k[:, :, int(perm[b * block + c]), 0] = val
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v


def _run(w, q, k, v, dense):
    dev = torch.device("cuda")
    g = F.Grid.make(w.grid, w.tile, w.block)
    nb = g.nb
    qp, kp, vp = (torch.empty((w.B, w.H, nb * w.block, w.d), dtype=torch.bfloat16, device=dev)
                  for _ in range(3))
    for x, y in ((q, qp), (k, kp), (v, vp)):
        F.fvattn_permute(x.to(dev), y, g)
    op = torch.zeros_like(qp)
    lse = torch.empty(qp.shape[:-1], dtype=torch.float32, device=dev)
    opk = F.FVATTN_OP_DENSE_FWD if dense else F.FVATTN_OP_SPARSE_FWD
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(opk, w.B, w.H, w.N, w.d, w.block), dev)
    idx = np.full((1, w.H, nb, nb), -1, dtype=np.int32)
    cnt = np.zeros((1, w.H, nb), dtype=np.int32)
    idx[..., :len(LIST)] = LIST
    cnt[...] = len(LIST)
    if dense:
        F.fvattn_dense_fwd(qp, kp, vp, op, w.N, w.block, ws, lse=lse)
    else:
        F.fvattn_sparse_fwd(qp, kp, vp, op, torch.from_numpy(idx).to(dev), torch.from_numpy(cnt).to(dev),
                            w.N, w.block, ws, lse=lse)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    mask = np.ones((1, w.H, nb, nb), dtype=bool)
    if not dense:
        mask[:] = False
        mask[..., LIST] = True
    return op.float().cpu().numpy(), lse.cpu().numpy(), mask


@pytest.mark.parametrize("dense", [False, True], ids=["sparse", "dense"])
@pytest.mark.parametrize("grid,tile,block", [((2, 32, 48), (1, 8, 8), 64),     # nb = 48 blocks of 64
                                              ((4, 32, 48), (2, 8, 8), 128)],   # nb = 48 blocks of 128
                         ids=["bs64", "bs128"])
def test_max_jumps_in_either_half(grid, tile, block, dense):
    w = S.Workload("rescale", 1, 2, 128, "bf16", grid, tile, block, 0.9, 1, seed=81, gen="gauss")
    q, k, v = _planted(w, block)
    out, lse, mask = _run(w, q, k, v, dense)
    perm = O.tile_order(*w.grid, *w.tile)
    qn, kn, vn = (O.permute(x.float().numpy(), perm, w.block) for x in (q, k, v))
    scale = 1.0 / math.sqrt(w.d)
    ref = O.masked_attention(qn, kn, vn, mask, w.N, w.block, scale)
    mx, mean = attention_errors(out[:, :, :w.N], ref[:, :, :w.N])
    assert np.all(np.isfinite(out[:, :, :w.N]))
    assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, (mx, mean)
    # the row log-sum-exp carries the running max through every rescale
    worst = 0.0
    for h in range(w.H):
        for i in range(0, mask.shape[2], 7):
            ref_l = O.row_lse(O.block_lse_rows(qn[0, h], kn[0, h], mask[0, h, i], w.N, w.block, scale, i))
            got = lse[0, h, i * w.block:i * w.block + ref_l.shape[0]]
            worst = max(worst, float(np.max(np.abs(got - ref_l) / np.maximum(1.0, np.abs(ref_l)))))
    assert worst <= 1e-4, worst
    big = float(np.max(lse[:, :, :w.N]))
    assert big > 100.0, big      # the planted logits were reached
    print(f"rescale {'dense' if dense else 'sparse'} bs {block}: max_abs {mx:.2e} mean_abs {mean:.2e} "
          f"lse rel err {worst:.1e}, max lse {big:.1f}")
