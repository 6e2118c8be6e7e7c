"""fp64 CPU oracle: 3-D tile permutation, block-mean pooling, block scores,
Top-p routing with a Top-k floor, per-head work, masked (block-sparse) and
dense softmax attention.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA product path
never imports this module, and this module imports nothing from it.

Every function restates one step of the method in plain NumPy fp64 with no
blocking, fusion or reordering beyond what the step's definition states. A
library primitive (``np.lexsort``, ``np.cumsum``, a matmul, ``np.exp``) may
serve as a step. Inputs are upcast to fp64; bf16 tensors reach this module as
float32 arrays holding the exact bf16 values.

Citations name the page and the section/equation:
  [FVAttn §2.1]  per-head block mask M_{h,i,j}, Top-k vs Top-p, Top-k floor
  [FVAttn §2.2]  Eq. (1): per-head workload L_h = mean_i sum_j M_{h,i,j}
  [FVAttn §3.1]  video-aware block order; pooled-Q/K block similarity; Top-p
                 CDF threshold; Top-k floor as a safety net
  [GSRS §3.2]    block-sparse attention skips unselected blocks
  [GSRS §5.2, §A.4] Top-p keeps the shortest descending prefix whose
                 cumulative importance reaches p
  [GSRS §5.3]    block importance sums to one over key blocks per query block
  [GSRS §A.1]    softmax attention evaluated block by block (online softmax)

Readings of points the pages leave open (each one is listed in the design notes):
  * block order: 3-D tiles (tt, th, tw) in tile-major raster order, raster
    order inside a tile; edge tiles are partial; the permuted sequence is cut
    into contiguous blocks of ``bs`` tokens and padded at the tail only.
  * score temperature: 1/sqrt(d), the attention scale.
  * pooling: mean over the valid tokens of a block only.
  * threshold: cumulative sum >= p ("reaches"); p >= 1 selects every block.
  * ties: descending score, then ascending block index.
  * floor: cnt = min(nbk, max(n_p, k_min)).
"""

from __future__ import annotations

import math

import numpy as np


def num_blocks(N: int, bs: int) -> int:
    """Number of blocks of ``bs`` tokens covering N tokens (last one may be partial)."""
    return -(-N // bs)


# --------------------------------------------------------------------------
# Step 1: video-aware token order [FVAttn §3.1], read as 3-D tiles
# --------------------------------------------------------------------------
def tile_order(T: int, Hh: int, W: int, tt: int, th: int, tw: int) -> np.ndarray:
    """Permutation of the T*Hh*W tokens of a (T, Hh, W) latent video grid.

    ``perm[pos]`` is the original token index ``n = (t*Hh + y)*W + x`` that
    lands at permuted position ``pos``. Tokens are sorted by the key
    ``(t//tt, y//th, x//tw, t%tt, y%th, x%tw)``: tiles in raster order over the
    tile grid, then raster order inside the tile. Built from explicit loops
    and a stable sort of the keys.
    """
    entries = []
    for t in range(T):
        for y in range(Hh):
            for x in range(W):
                key = (t // tt, y // th, x // tw, t % tt, y % th, x % tw)
                entries.append((key, (t * Hh + y) * W + x))
    entries.sort(key=lambda e: e[0])  # Python's sort is stable; keys are unique anyway
    return np.fromiter((n for _, n in entries), dtype=np.int64, count=len(entries))


def permute(x: np.ndarray, perm: np.ndarray, bs: int) -> np.ndarray:
    """Gather ``x[..., N, d]`` into tile order, padded with zero rows to nb*bs."""
    N = len(perm)
    npad = num_blocks(N, bs) * bs
    y = np.zeros(x.shape[:-2] + (npad, x.shape[-1]), dtype=x.dtype)
    y[..., :N, :] = x[..., perm, :]
    return y


def inverse_permute(y: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Scatter ``y[..., Npad, d]`` (tile order) back to original order; pad rows dropped."""
    N = len(perm)
    x = np.empty(y.shape[:-2] + (N, y.shape[-1]), dtype=y.dtype)
    x[..., perm, :] = y[..., :N, :]
    return x


# --------------------------------------------------------------------------
# Step 2: block-mean pooling and block scores [FVAttn §3.1, §2.1; GSRS §5.3]
# --------------------------------------------------------------------------
def block_mean_pool(xp: np.ndarray, N: int, bs: int) -> np.ndarray:
    """Mean of the valid tokens of each block of a permuted ``xp[..., Npad, d]``."""
    xp = np.asarray(xp, dtype=np.float64)
    nb = num_blocks(N, bs)
    out = np.empty(xp.shape[:-2] + (nb, xp.shape[-1]), dtype=np.float64)
    for i in range(nb):
        lo, hi = i * bs, min((i + 1) * bs, N)
        out[..., i, :] = xp[..., lo:hi, :].sum(axis=-2) / (hi - lo)
    return out


def block_scores(qbar: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """Normalized block importance s_{i,j} = softmax_j(scale * qbar_i . kbar_j).

    The max is subtracted before exponentiation. Each row sums to one, which is
    what Top-p accumulates.
    """
    logits = np.matmul(np.asarray(qbar, np.float64),
                       np.swapaxes(np.asarray(kbar, np.float64), -1, -2)) * scale
    logits = logits - logits.max(axis=-1, keepdims=True)
    e = np.exp(logits)
    return e / e.sum(axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# Step 3: Top-p selection with a Top-k floor [FVAttn §2.1, §3.1; GSRS §5.2, §A.4]
# --------------------------------------------------------------------------
def topp_topk_select(s: np.ndarray, p: float, k_min: int):
    """Select key blocks for one query block from its importance row ``s``.

    Returns ``(order, cnt)``: ``order`` ranks all key blocks by descending
    importance (ties: lower block index first); the selected set is
    ``order[:cnt]``. n_p is the smallest c whose cumulative importance over
    the first c ranked blocks is >= p (every block when p >= 1 or when no
    prefix reaches p); the floor gives cnt = min(nbk, max(n_p, k_min)).
    """
    s = np.asarray(s, dtype=np.float64)
    nbk = s.shape[-1]
    order = np.lexsort((np.arange(nbk), -s))
    if p >= 1.0:
        n_p = nbk
    else:
        cum = np.cumsum(s[order])
        hit = np.nonzero(cum >= p)[0]
        n_p = int(hit[0]) + 1 if hit.size else nbk
    cnt = min(nbk, max(n_p, int(k_min)))
    return order, cnt


def selection_mask(order: np.ndarray, cnt: np.ndarray) -> np.ndarray:
    """Block mask M[..., i, j] in {0,1} from ranked orders and counts [FVAttn §2.1]."""
    order = np.asarray(order)
    cnt = np.asarray(cnt)
    nbk = order.shape[-1]
    rank_ok = np.arange(nbk) < cnt[..., None]          # [..., nb, nbk] over ranks
    mask = np.zeros(order.shape, dtype=bool)
    np.put_along_axis(mask, order, rank_ok, axis=-1)
    return mask


def head_work(cnt: np.ndarray) -> np.ndarray:
    """Selected block pairs per head, sum_i cnt_i = nb * L_h of [FVAttn §2.2, Eq. (1)]."""
    return np.asarray(cnt, dtype=np.int64).sum(axis=-1)


def route(q, k, grid, bs: int, p: float, k_min: int, scale: float | None = None, perm=None):
    """Routing front end for q, k ``[B, H, N, d]`` in original token order.

    Steps: tile permutation (or the explicit token order ``perm``, e.g. the
    Hilbert order, when given), block-mean pooling of Q and K, block scores, and
    per-row Top-p with the Top-k floor. Returns a dict with ``perm``,
    ``qbar``, ``kbar``, ``scores`` (fp64 [B,H,nb,nb]), ``order`` (int64
    [B,H,nb,nb]), ``cnt`` (int64 [B,H,nb]) and ``head_work`` (int64 [B,H]).
    Heads are processed one at a time to bound memory.
    """
    T, Hh, W, tt, th, tw = grid
    if perm is None:
        perm = tile_order(T, Hh, W, tt, th, tw)
    B, H, N, d = q.shape
    if N != len(perm):
        raise ValueError("N must equal T*Hh*W")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nb = num_blocks(N, bs)
    qbar = np.empty((B, H, nb, d))
    kbar = np.empty((B, H, nb, d))
    scores = np.empty((B, H, nb, nb))
    order = np.empty((B, H, nb, nb), dtype=np.int64)
    cnt = np.empty((B, H, nb), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            qp = permute(np.asarray(q[b, h], np.float64), perm, bs)
            kp = permute(np.asarray(k[b, h], np.float64), perm, bs)
            qbar[b, h] = block_mean_pool(qp, N, bs)
            kbar[b, h] = block_mean_pool(kp, N, bs)
            scores[b, h] = block_scores(qbar[b, h], kbar[b, h], scale)
            for i in range(nb):
                order[b, h, i], cnt[b, h, i] = topp_topk_select(scores[b, h, i], p, k_min)
    return dict(perm=perm, qbar=qbar, kbar=kbar, scores=scores, order=order,
                cnt=cnt, head_work=head_work(cnt))


# --------------------------------------------------------------------------
# Step 4: block-sparse attention [FVAttn §2.1; GSRS §3.2, §A.1]
# --------------------------------------------------------------------------
def _softmax_attend(qr: np.ndarray, kk: np.ndarray, vv: np.ndarray, scale: float) -> np.ndarray:
    logits = (qr @ kk.T) * scale
    logits = logits - logits.max(axis=-1, keepdims=True)
    w = np.exp(logits)
    w = w / w.sum(axis=-1, keepdims=True)
    return w @ vv


def masked_attention_rows(qp, kp, vp, mask_row, N: int, bs: int, scale: float, i: int) -> np.ndarray:
    """Output rows of query block ``i`` of one head (permuted layout, ``[Npad, d]`` inputs).

    Each query token of block i takes a softmax over the valid keys of the
    selected key blocks only (mask_row[j] true), then weights V. Returns the
    ``min(bs, N - i*bs)`` valid rows.
    """
    qp = np.asarray(qp, np.float64)
    kp = np.asarray(kp, np.float64)
    vp = np.asarray(vp, np.float64)
    lo, hi = i * bs, min((i + 1) * bs, N)
    cols = np.concatenate([np.arange(j * bs, min((j + 1) * bs, N))
                           for j in np.nonzero(np.asarray(mask_row))[0]])
    return _softmax_attend(qp[lo:hi], kp[cols], vp[cols], scale)


def masked_attention(qp, kp, vp, mask, N: int, bs: int, scale: float, blocks=None) -> np.ndarray:
    """Block-sparse attention over permuted ``[B, H, Npad, d]`` tensors.

    ``mask`` is [B, H, nb, nb] bool. Returns fp64 [B, H, Npad, d]; pad rows
    and query blocks not listed in ``blocks`` (an iterable of (b, h, i); all
    when None) are left at zero.
    """
    B, H, npad, d = qp.shape
    nb = num_blocks(N, bs)
    out = np.zeros((B, H, npad, d))
    todo = blocks if blocks is not None else [(b, h, i) for b in range(B) for h in range(H) for i in range(nb)]
    for (b, h, i) in todo:
        rows = masked_attention_rows(qp[b, h], kp[b, h], vp[b, h], mask[b, h, i], N, bs, scale, i)
        out[b, h, i * bs:i * bs + rows.shape[0]] = rows
    return out


def dense_attention(q, k, v, scale: float) -> np.ndarray:
    """Textbook softmax(q k^T * scale) v per (b, h) in fp64, any token order."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    out = np.empty(q.shape[:-1] + (v.shape[-1],))
    for idx in np.ndindex(*q.shape[:-2]):
        out[idx] = _softmax_attend(q[idx], k[idx], v[idx], scale)
    return out
