"""GPU parity of the low-precision V path: fvattn_quantize_v bit for bit against
the oracle's per-channel E4M3 quantization, and fvattn_sparse_fwd_fp8v /
fvattn_dense_fwd_fp8v against the oracle's masked attention over the
dequantized V, run on the GPU's own mask. [FVAttn §3.4: V is quantized on the
GPU before attention.]

Tolerance of the attention output, derived from the kernel's arithmetic. Work
in units where the row's largest exp(logit - max) is 1: P_j <= 1, W = sum P_j,
w_j = P_j / W the oracle's weights, O = sum w_j V^_j the oracle's output.
  * The kernel multiplies E4M3(P_j) by the E4M3 codes of V. P is formed
    relative to m_run - 4 with m_run in [max - 4, max], so in these units the
    rounding error is |e_j| <= 2^-4 P_j (normal range) + 2^-14 (subnormal step).
  * With L = sum E4M3(P_j) as the normaliser (the kernel sums the rounded
    values), the output is sum (P_j + e_j) V^_j / (W + sum e_j), and because
    sum w_j (V^_j - O) = 0 the error is exactly sum_j e_j (V^_j - O) / (W + sum e).
    Bound (per row r, channel c):
        B1 = sum_j (2^-4 w_j + 2^-14 / W) |V^_jc - O_c| / (1 - 2^-4 - n 2^-14 / W)
  * L is summed as exact f16 pairs over 16 keys (at most 8 rounded additions,
    relative error <= 2^-8), the output is rounded to bf16 (2^-9 relative):
        B2 = (2^-8 + 2^-8) |O_c|
  * The tensor cores accumulate the 8-bit products; a relative accumulation
    error of up to 2^-10 of the magnitudes is allowed for:
        B3 = 2^-10 sum_j w_j |V^_jc|
  Gate 1 (every element of the rows checked): |err| <= B1 + B2 + B3 + 1e-6,
  where B1 is finite (n 2^-14 / W < 1 - 2^-4); rows where it is not are left to
  gate 2.
  Gate 2 (overall): with the rounding errors independent and of relative RMS at
  most 2^-4 / sqrt(3), the predicted variance of an element is
        s^2 = sum_j ((2^-4/sqrt 3)^2 w_j^2 + (2^-14/W)^2 / 3) (V^_jc - O_c)^2,
  and the RMS of the errors must stay below 2 sqrt(mean s^2) + 2^-8 RMS(O) + 1e-4.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from oracle import lowprec_oracle as Lp
from parity import mask_from_lists
from test_gpu_parity import BS64, ODD128, PEAKY, SINGLE, _route_gpu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_video_b200 as F

REL_P = 2.0 ** -4
SUB_P = 2.0 ** -14


def _np(t):
    return t.detach().float().cpu().numpy()


def _perm(w):
    return O.tile_order(*w.grid, *w.tile)


def _quant_gpu(w, vp):
    dev = vp.device
    vq = torch.full(vp.shape, 0xA5, dtype=torch.uint8, device=dev)
    vs = torch.full((w.B, w.H, w.d), float("nan"), dtype=torch.float32, device=dev)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_QUANT_V, w.B, w.H, w.N, w.d, w.block), dev)
    F.fvattn_quantize_v(vp, vq, vs, w.N, w.block, ws)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    return vq, vs


def _same_codes(a, b):
    """Equal codes, with +0 (0x00) and -0 (0x80) counted as the same value."""
    return (a == b) | (((a & 0x7F) == 0) & ((b & 0x7F) == 0))


def _inputs(w):
    """GPU tensors (original order, permuted) and the oracle's own permutation of them."""
    q, k, v = S.make_qkv(w, device="cuda")
    grid = F.Grid.make(w.grid, w.tile, w.block)
    vp = torch.empty((w.B, w.H, grid.nb * w.block, w.d), dtype=v.dtype, device="cuda")
    F.fvattn_permute(v, vp, grid)
    perm = _perm(w)
    ref = [O.permute(_np(x), perm, w.block) for x in (q, k, v)]
    return q, k, v, vp, ref


@pytest.mark.parametrize("w", [ODD128, BS64, PEAKY, SINGLE, S.WORKLOADS["wan1.3b-480p"]],
                         ids=lambda w: w.name)
def test_quantize_v_matches_oracle(w):
    _, _, _, vp, (_, _, vref) = _inputs(w)
    vq, vs = _quant_gpu(w, vp)
    codes, scale = Lp.quantize_v(vref, w.N)
    got = vq.cpu().numpy()
    same = _same_codes(got, codes)
    assert same.all(), (np.argwhere(~same)[:5], got[~same][:5], codes[~same][:5])
    assert np.array_equal(vs.cpu().numpy(), scale)
    print(f"{w.name}: {got.size} codes, {int(((got & 0x7F) == 0).sum())} zeros, "
          f"{int((np.abs(Lp.e4m3_decode(got)) == 448).sum())} at +-448")


@pytest.mark.parametrize("w", [ODD128, BS64, SINGLE, S.WORKLOADS["wan1.3b-480p"]], ids=lambda w: w.name)
@pytest.mark.parametrize("order", ["tiles", "hilbert"])
def test_permute_quantize_v_equals_permute_then_quantize(w, order):
    """The fused call gives the codes and scales of fvattn_permute + fvattn_quantize_v,
    bit for bit (including +-0 and the pad rows), and those of the oracle."""
    q, k, v = S.make_qkv(w, device="cuda")
    table = F.fvattn_hilbert_table(w.grid, w.block) if order == "hilbert" else None
    grid = F.Grid.make(w.grid, w.tile, w.block, table=table)
    npad = grid.nb * w.block
    vp = torch.empty((w.B, w.H, npad, w.d), dtype=v.dtype, device="cuda")
    F.fvattn_permute(v, vp, grid)
    vq2, vs2 = _quant_gpu(w, vp)
    vq = torch.full((w.B, w.H, npad, w.d), 0xA5, dtype=torch.uint8, device="cuda")
    vs = torch.full((w.B, w.H, w.d), float("nan"), dtype=torch.float32, device="cuda")
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_QUANT_V, w.B, w.H, w.N, w.d, w.block), "cuda")
    for _ in range(2):      # the workspace's maxima are cleared by every call
        F.fvattn_permute_quantize_v(v, grid, vq, vs, ws)
        assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
        assert torch.equal(vq, vq2) and torch.equal(vs, vs2)
    perm = table.cpu().numpy().astype(np.int64) if table is not None else _perm(w)
    codes, scale = Lp.quantize_v(O.permute(_np(v), perm, w.block), w.N)
    assert _same_codes(vq.cpu().numpy(), codes).all()
    assert np.array_equal(vs.cpu().numpy(), scale)


def test_quantize_v_sampled_720p_heads():
    # the 14B-720p V, full call; the oracle checks two heads completely
    w = S.WORKLOADS["wan14b-720p"]
    q, k, v = S.make_qkv(w, device="cuda")
    del q, k
    grid = F.Grid.make(w.grid, w.tile, w.block)
    vp = torch.empty((w.B, w.H, grid.nb * w.block, w.d), dtype=v.dtype, device="cuda")
    F.fvattn_permute(v, vp, grid)
    vq, vs = _quant_gpu(w, vp)
    perm = _perm(w)
    for h in (0, w.H - 1):
        vref = O.permute(_np(v[:, h:h + 1]), perm, w.block)
        codes, scale = Lp.quantize_v(vref, w.N)
        assert _same_codes(vq[:, h:h + 1].cpu().numpy(), codes).all(), h
        assert np.array_equal(vs[:, h:h + 1].cpu().numpy(), scale), h


def test_quantize_v_special_channels():
    # a zero channel, a channel holding one huge outlier, a channel of ties
    w = S.Workload("quant-special", 1, 2, 128, "bf16", (3, 8, 12), (1, 8, 8), 64, 0.9, 1, seed=41)
    _, _, _, vp, (_, _, vref) = _inputs(w)
    pattern = np.resize(np.array([1.0, 0.09375, -0.25, 0.5], np.float32), w.N)
    vref = vref.copy()
    vref[:, :, :, 3] = 0.0
    vref[0, 1, 5, 7] = 29952.0                               # a bf16 value far above the rest
    vref[:, 0, : w.N, 9] = pattern
    vp[:, :, :, 3] = 0.0
    vp[0, 1, 5, 7] = 29952.0
    vp[:, 0, : w.N, 9] = torch.from_numpy(pattern).to(vp.dtype).cuda()
    assert np.array_equal(_np(vp), vref)
    vq, vs = _quant_gpu(w, vp)
    codes, scale = Lp.quantize_v(vref, w.N)
    assert _same_codes(vq.cpu().numpy(), codes).all()
    assert np.array_equal(vs.cpu().numpy(), scale)
    assert float(vs[0, 0, 3]) == 0.0 and int(vq[0, :, :, 3].abs().sum()) == 0
    assert int(vq[0, 0, 1, 9]) == 0x62                       # 42 rounds to 40 (even mantissa)


def _fp8_attn(w, qp, kp, vq, vs, kv_idx=None, kv_cnt=None, lse=False):
    dev = qp.device
    op = torch.full_like(qp, float("nan"))
    lse_t = torch.empty(qp.shape[:-1], dtype=torch.float32, device=dev) if lse else None
    opk = F.FVATTN_OP_DENSE_FWD if kv_idx is None else F.FVATTN_OP_SPARSE_FWD
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(opk, w.B, w.H, w.N, w.d, w.block), dev)
    if kv_idx is None:
        F.fvattn_dense_fwd_fp8v(qp, kp, vq, vs, op, w.N, w.block, ws, lse=lse_t)
    else:
        F.fvattn_sparse_fwd_fp8v(qp, kp, vq, vs, op, kv_idx, kv_cnt, w.N, w.block, ws, lse=lse_t)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    return op, lse_t


def _check_fp8_rows(w, qn, kn, vh, mask, out, lse, rows):
    """Gates 1 and 2 of the module docstring over the valid rows of the listed
    (b, h, i) query blocks. Returns (max err, rms err, predicted rms, rows gated)."""
    sm = 1.0 / math.sqrt(w.d)
    sq_err, sq_pred, sq_out, n_el = 0.0, 0.0, 0.0, 0
    worst, gated = 0.0, 0
    for (b, h, i) in rows:
        cols, wts = Lp.masked_softmax_weights(qn[b, h], kn[b, h], mask[b, h, i], w.N, w.block, sm, i)
        vv = vh[b, h, cols]                                   # [n, d]
        ref = wts @ vv                                        # [rows, d]
        lo = i * w.block
        got = out[b, h, lo:lo + ref.shape[0]].astype(np.float64)
        err = np.abs(got - ref)
        n = len(cols)
        Wu = 1.0 / wts.max(axis=1)                            # W in units of the row max
        denom = 1.0 - REL_P - n * SUB_P / Wu
        # L = W (1 + eps) with |eps| <= 1 - denom, summed with relative error <= 2^-8
        lse_tol = np.where(denom > 0, -np.log(np.maximum(denom, 1e-300)) + 2.0 ** -7 + 1e-5, np.inf)
        for r in range(ref.shape[0]):
            dev = np.abs(vv - ref[r])                         # |V^_j - O| [n, d]
            b1 = ((REL_P * wts[r] + SUB_P / Wu[r]) @ dev) / denom[r] if denom[r] > 0 else np.inf
            b2 = 2.0 ** -7 * np.abs(ref[r])
            b3 = 2.0 ** -10 * (wts[r] @ np.abs(vv))
            bound = b1 + b2 + b3 + 1e-6
            assert np.all(err[r] <= bound), (b, h, i, r, float((err[r] - bound).max()))
            gated += int(np.isfinite(b1).all())
            var = ((REL_P ** 2 / 3) * wts[r] ** 2 + (SUB_P / Wu[r]) ** 2 / 3) @ dev ** 2
            sq_pred += float(var.sum())
        sq_err += float((err ** 2).sum())
        sq_out += float((ref ** 2).sum())
        n_el += err.size
        worst = max(worst, float(err.max()))
        if lse is not None:
            logits = (qn[b, h, lo:lo + ref.shape[0]].astype(np.float64) @ kn[b, h, cols].T.astype(np.float64)) * sm
            mx = logits.max(axis=1)
            ref_lse = mx + np.log(np.exp(logits - mx[:, None]).sum(axis=1))
            assert np.all(np.abs(lse[b, h, lo:lo + ref.shape[0]] - ref_lse) <= lse_tol), (b, h, i)
    rms = math.sqrt(sq_err / n_el)
    pred = math.sqrt(sq_pred / n_el)
    assert rms <= 2.0 * pred + 2.0 ** -8 * math.sqrt(sq_out / n_el) + 1e-4, (rms, pred)
    return worst, rms, pred, gated


@pytest.mark.parametrize("w", [ODD128, BS64, PEAKY, SINGLE], ids=lambda w: w.name)
@pytest.mark.parametrize("dense", [False, True], ids=["sparse", "dense"])
def test_fp8v_attention_matches_oracle(w, dense):
    q, k, _, vp, (qn, kn, vn) = _inputs(w)
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    assert np.array_equal(_np(qp), qn) and np.array_equal(_np(kp), kn)
    vq, vs = _quant_gpu(w, vp)
    codes, scale = Lp.quantize_v(vn, w.N)
    vh = Lp.dequantize_v(codes, scale)
    nb = grid.nb
    if dense:
        op, lse = _fp8_attn(w, qp, kp, vq, vs, lse=True)
        mask = np.ones((w.B, w.H, nb, nb), bool)
    else:
        op, lse = _fp8_attn(w, qp, kp, vq, vs, kv_idx, kv_cnt, lse=True)
        mask = mask_from_lists(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), nb)
    out = _np(op)
    rows = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(nb)]
    worst, rms, pred, gated = _check_fp8_rows(w, qn, kn, vh, mask, out, lse.cpu().numpy(), rows)
    # context: the same call against attention on the unquantized V
    ref_v = O.masked_attention(qn, kn, vn, mask, w.N, w.block, 1.0 / math.sqrt(w.d))
    full = np.abs(out[:, :, :w.N] - ref_v[:, :, :w.N])
    print(f"{w.name} {'dense' if dense else 'sparse'}: density {mask.mean():.3f} max err {worst:.2e} "
          f"rms {rms:.2e} (predicted {pred:.2e}); rows gated {gated}; vs unquantized V: "
          f"max {full.max():.2e} mean {full.mean():.2e}")


def test_fp8v_zero_channel_gives_zero_output():
    w = ODD128
    q, k, _, vp, _ = _inputs(w)
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    vp[:, :, :, 17] = 0.0
    vq, vs = _quant_gpu(w, vp)
    op, _ = _fp8_attn(w, qp, kp, vq, vs, kv_idx, kv_cnt)
    assert torch.all(op[:, :, : w.N, 17] == 0)
    assert torch.isfinite(op[:, :, : w.N]).all()


def test_fp8v_path_sampled_720p():
    # the full 14B-720p call through FVAttnPath with the E4M3 V, oracle on sampled
    # query blocks (gate 2 at this size; gate 1 where it is finite)
    w = S.WORKLOADS["wan14b-720p"]
    q, k, v = S.make_qkv(w, device="cuda")
    path = F.FVAttnPath(w.B, w.H, w.grid, w.tile, w.block, w.d, torch.bfloat16, w.p, w.k_min, v_format="e4m3")
    out = path(q, k, v)
    assert F.fvattn_workspace_status(path.ws_attn) == F.FVATTN_OK
    perm = _perm(w)
    nb = path.nb
    cnt = path.kv_cnt.cpu().numpy()
    mask = mask_from_lists(path.kv_idx.cpu().numpy(), cnt, nb)
    rng = np.random.default_rng(9)
    heads = [int(cnt[0].sum(-1).argmax()), int(cnt[0].sum(-1).argmin()), int(rng.integers(0, w.H))]
    rows = []
    for h in heads:
        rows += [(0, h, int(i)) for i in rng.integers(0, nb, 2)]
    rows.append((0, heads[0], nb - 1))
    qn = O.permute(_np(q[:, heads]), perm, w.block)
    kn = O.permute(_np(k[:, heads]), perm, w.block)
    vn = O.permute(_np(v[:, heads]), perm, w.block)
    codes, scale = Lp.quantize_v(vn, w.N)
    vh = Lp.dequantize_v(codes, scale)
    outp = O.permute(_np(out[:, heads]), perm, w.block)
    local = [(0, heads.index(h), i) for (_, h, i) in rows]
    worst, rms, pred, gated = _check_fp8_rows(w, qn, kn, vh, mask[:, heads], outp, None, local)
    print(f"wan14b-720p fp8 V: {len(rows)} query blocks, max err {worst:.2e} rms {rms:.2e} "
          f"(predicted {pred:.2e}); rows gated {gated}")


def test_fp8v_block_lse_gives_importance():
    # block log-sum-exps of the E4M3 launch feed the GSRS importance: rows sum to one (block
    # and row sums come from the same rounded P) and each entry stays within the P rounding
    # of the exact importance. Each is a mean of ratios of sums of rounded P; with the
    # relative rounding r = 2^-4 + N 2^-14 (normal steps, plus the subnormal steps of up to
    # N keys against a row sum >= 1), a ratio is off by at most 2r / (1 - r) relative, plus
    # the subnormal steps of one block, at most 128 * 2^-14 = 2^-7.
    w = ODD128
    q, k, _, vp, (qn, kn, _) = _inputs(w)
    grid, qp, kp, kv_idx, kv_cnt, _ = _route_gpu(w, q, k)
    vq, vs = _quant_gpu(w, vp)
    nb = grid.nb
    lse = torch.empty(qp.shape[:-1], dtype=torch.float32, device="cuda")
    blse = torch.full((w.B, w.H, nb, qp.shape[2]), 12345.0, dtype=torch.float32, device="cuda")
    op = torch.empty_like(qp)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_SPARSE_FWD, w.B, w.H, w.N, w.d, w.block), "cuda")
    F.fvattn_sparse_fwd_fp8v(qp, kp, vq, vs, op, kv_idx, kv_cnt, w.N, w.block, ws, lse=lse, block_lse=blse)
    assert F.fvattn_workspace_status(ws) == F.FVATTN_OK
    imp = torch.empty((w.B, w.H, nb, nb), dtype=torch.float32, device="cuda")
    wsd = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_DIAG, w.B, w.H, w.N, w.d, w.block), "cuda")
    F.fvattn_block_importance(blse, lse, imp, w.N, w.block, wsd, kv_idx=kv_idx, kv_cnt=kv_cnt)
    assert F.fvattn_workspace_status(wsd) == F.FVATTN_OK
    got = imp.cpu().numpy()
    mask = mask_from_lists(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), nb)
    ref = O.block_importance(qn, kn, mask, w.N, w.block, 1.0 / math.sqrt(w.d))
    assert np.abs(got.sum(-1) - 1.0).max() <= 1e-4
    assert np.all(got[~mask] == 0.0)
    r = REL_P + w.N * SUB_P
    assert np.all(np.abs(got - ref) <= 2 * r / (1 - r) * ref + 2.0 ** -7), np.abs(got - ref).max()
    print(f"fp8 V importance: max |d| {np.abs(got - ref).max():.2e}, mean |d| {np.abs(got - ref)[mask].mean():.2e}")
