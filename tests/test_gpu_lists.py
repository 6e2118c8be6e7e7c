"""GPU: attention over hand-made KV lists, against the oracle's masked attention on the
oracle's own permutation of the same seeded inputs [FVAttn §2.1: only the selected
(query block, key block) pairs are evaluated].

The lists are built so that, in the 64-token kernel's four-query-block units, one tile
slot (two query blocks) has no selected entry in many 128-key steps while the other
does, the only members of a slot sit at the two ends of the union, and union entries
straddle the 32-entry windows in which the kernel's MMA warp reads slot membership.
The same lists run at 128-token blocks on a grid of the same block count."""

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


def _lists(nb, H, seed):
    """[1, H, nb, nb] int32 lists and [1, H, nb] counts (host side, deterministic)."""
    rng = np.random.default_rng(seed)
    idx = np.full((1, H, nb, nb), -1, dtype=np.int32)
    cnt = np.zeros((1, H, nb), dtype=np.int32)
    for h in range(H):
        for i in range(nb):
            g, r = divmod(i, 4)
            if h == 0:
                # four-block units: block 0 of a unit takes the first and last key block,
                # block 1 a single moving one, blocks 2 and 3 (the other slot) entries
                # around the 32-entry window edge only
                sel = {0: [0, nb - 1], 1: [g % nb], 2: [min(33, nb - 1)], 3: [31, min(32, nb - 1)]}[r]
            else:
                k = int(rng.integers(1, 6))
                sel = sorted(set(int(x) for x in rng.choice(nb, size=k, replace=False)))
            sel = sorted(set(sel))
            idx[0, h, i, :len(sel)] = sel
            cnt[0, h, i] = len(sel)
    return idx, cnt


@pytest.mark.parametrize("grid,tile,block", [((2, 32, 48), (1, 8, 8), 64),     # nb = 48 blocks of 64
                                              ((4, 32, 48), (2, 8, 8), 128)],   # nb = 48 blocks of 128
                         ids=["bs64", "bs128"])
def test_attention_over_hand_made_lists(grid, tile, block):
    w = S.Workload("lists", 1, 2, 128, "bf16", grid, tile, block, 0.9, 1, seed=71)
    dev = torch.device("cuda")
    q, k, v = S.make_qkv(w, device=dev)
    g = F.Grid.make(w.grid, w.tile, w.block)
    nb = g.nb
    assert nb == 48
    idx_np, cnt_np = _lists(nb, w.H, seed=72)
    qp, kp, vp = (torch.empty((w.B, w.H, nb * w.block, w.d), dtype=q.dtype, device=dev) for _ in range(3))
    for x, y in ((q, qp), (k, kp), (v, vp)):
        F.fvattn_permute(x, y, g)
    op = torch.zeros_like(qp)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_SPARSE_FWD, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_sparse_fwd(qp, kp, vp, op, torch.from_numpy(idx_np).to(dev), torch.from_numpy(cnt_np).to(dev),
                        w.N, w.block, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    mask = np.zeros((1, w.H, nb, nb), dtype=bool)
    for h in range(w.H):
        for i in range(nb):
            mask[0, h, i, idx_np[0, h, i, :cnt_np[0, h, i]]] = True
    to_np = lambda t: t.float().cpu().numpy()
    perm = O.tile_order(*w.grid, *w.tile)
    ref = O.masked_attention(*(O.permute(to_np(x), perm, w.block) for x in (q, k, v)), mask, w.N, w.block,
                             1.0 / math.sqrt(w.d))
    mx, mean = attention_errors(to_np(op)[:, :, :w.N], ref[:, :, :w.N])
    assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, (mx, mean)
    # every row attends something: no row is left at zero
    assert np.all(np.abs(to_np(op)[:, :, :w.N]).sum(-1) > 0)
    print(f"hand-made lists bs {block}: density {mask.mean():.3f} max_abs {mx:.2e} mean_abs {mean:.2e}")
