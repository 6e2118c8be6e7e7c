"""fvattn_route_noalloc against fvattn_route, through the C ABI.

Some callers cannot allocate device memory where they route: an engine plugin
that owns all device memory and has no scratch buffer to hand over, or a hot
loop where cudaMalloc would synchronize the device. For them the library keeps
a static 96 MiB device array as the router's scratch. These tests check that
routing through that array gives exactly what the workspace entry point gives,
on two calls in a row (the second call finds the first call's leftovers in
the shared array), and that sizes beyond the array are refused.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test; it does not depend on them.
"""

import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_video_b200 as F
import synthetic as S


def _route_both(w, seed_shift):
    dev = torch.device("cuda")
    q, k, _ = S.make_qkv(w.replace(seed=w.seed + seed_shift), device=dev)
    grid = F.Grid.make(w.grid, w.tile, w.block)
    nb, npad = grid.nb, grid.nb * w.block
    outs = []
    for use_scratch in (False, True):
        qp = torch.zeros((w.B, w.H, npad, w.d), dtype=q.dtype, device=dev)
        kp = torch.zeros_like(qp)
        idx = torch.full((w.B, w.H, nb, nb), -1, dtype=torch.int32, device=dev)
        cnt = torch.zeros((w.B, w.H, nb), dtype=torch.int32, device=dev)
        hw = torch.zeros((w.B, w.H), dtype=torch.int64, device=dev)
        if use_scratch:
            st = F._lib.fvattn_route_noalloc(
                F._ptr(q), F._ptr(k), w.B, w.H, w.N, w.d, F._dtype_code(q), ctypes.byref(grid),
                float(w.p), int(w.k_min), F._ptr(qp), F._ptr(kp), F._ptr(idx), F._ptr(cnt),
                F._ptr(hw), F._stream(None))
            assert st == F.FVATTN_OK, F.fvattn_status_string(st)
        else:
            ws = F.alloc_workspace(
                F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, w.B, w.H, w.N, w.d, w.block), dev)
            F.fvattn_route(q, k, grid, w.p, w.k_min, idx, cnt, hw, ws, qp_out=qp, kp_out=kp)
        torch.cuda.synchronize()
        outs.append((qp, kp, idx.cpu().numpy(), cnt.cpu().numpy(), hw.cpu().numpy()))
    return outs


@pytest.mark.gpu
def test_noalloc_route_matches_workspace_route_on_two_calls():
    # two calls in a row, with different inputs, through the shared scratch
    for shift, w in ((0, S.WORKLOADS["wan1.3b-480p"]), (77, S.WORKLOADS["wan14b-480p"])):
        (qp_a, kp_a, idx_a, cnt_a, hw_a), (qp_b, kp_b, idx_b, cnt_b, hw_b) = _route_both(w, shift)
        assert torch.equal(qp_a, qp_b) and torch.equal(kp_a, kp_b)
        assert np.array_equal(cnt_a, cnt_b)
        assert np.array_equal(hw_a, hw_b)
        valid = np.arange(idx_a.shape[-1]) < cnt_a[..., None]
        assert np.array_equal(np.where(valid, idx_a, -1), np.where(valid, idx_b, -1))


def test_noalloc_route_refuses_sizes_beyond_its_scratch():
    # 40 heads x 1,182 blocks of 64 tokens x d=128 need 48 MB of block means and 224 MB of scores.
    grid = F.Grid.make((21, 45, 80), (1, 8, 8), 64)
    need = F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, 1, 40, grid.N, 128, 64)
    assert need > (96 << 20)
    fake = 1 << 20
    st = F._lib.fvattn_route_noalloc(fake, fake, 1, 40, grid.N, 128, F.FVATTN_BF16, ctypes.byref(grid),
                                     0.9, 4, None, None, fake, fake, fake, None)
    assert st == F.FVATTN_ERR_WORKSPACE
