"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments with a status before any launch."""

import ctypes
import os
import re

import pytest

import block_sparse_attention_video_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"FVATTN_API\s+[\w\s\*]+?\b(fvattn_\w+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_four_calls_and_helpers():
    decl = _declared_symbols()
    for name in ("fvattn_permute", "fvattn_route", "fvattn_sparse_fwd", "fvattn_dense_fwd",
                 "fvattn_block_importance", "fvattn_attention_recall",
                 "fvattn_workspace_bytes", "fvattn_workspace_status", "fvattn_status_string"):
        assert name in decl


@pytest.mark.parametrize("name", _declared_symbols())
def test_library_exports_every_declared_symbol(name):
    lib = ctypes.CDLL(F.LIB_PATH)
    assert hasattr(lib, name)


def test_status_strings():
    for code in range(6):
        assert F.fvattn_status_string(code)
    assert F.fvattn_status_string(99) == "unknown status"


def test_workspace_bytes():
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_DENSE_FWD, 1, 40, 75600, 128, 128) == 256
    nb = 591
    route = F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, 1, 40, 75600, 128, 128)
    assert route >= 256 + 2 * 40 * nb * 128 * 4
    sparse = F.fvattn_workspace_bytes(F.FVATTN_OP_SPARSE_FWD, 1, 40, 75600, 128, 128)
    assert sparse >= 256 + 40 * nb * 4 + 40 * 12
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, 1, 40, 75600, 96, 128) == 0   # bad d
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, 1, 40, 75600, 128, 32) == 0   # bad block
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_ROUTE, 0, 40, 75600, 128, 128) == 0


FAKE = 1 << 20          # 16-byte aligned non-null address; never dereferenced (validation fails first)


def _grid(**kw):
    g = dict(T=4, Hh=8, W=8, tt=1, th=8, tw=8, block=64)
    g.update(kw)
    return F.Grid(g["T"], g["Hh"], g["W"], g["tt"], g["th"], g["tw"], g["block"])


def _permute(x=FAKE, y=FAKE * 4, N=256, d=64, dt=F.FVATTN_FP32, grid=None):
    g = grid if grid is not None else _grid()
    return F._lib.fvattn_permute(x, y, 1, 2, N, d, dt, ctypes.byref(g), 0, None)


@pytest.mark.parametrize("kw, status", [
    (dict(x=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(y=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(x=FAKE + 4), F.FVATTN_ERR_INVALID_ARG),          # misaligned
    (dict(N=255), F.FVATTN_ERR_INVALID_ARG),               # N != T*Hh*W
    (dict(d=96), F.FVATTN_ERR_INVALID_ARG),
    (dict(dt=7), F.FVATTN_ERR_INVALID_ARG),
    (dict(grid=_grid(tt=0)), F.FVATTN_ERR_INVALID_ARG),
    (dict(grid=_grid(block=32)), F.FVATTN_ERR_INVALID_ARG),
    (dict(y=FAKE + 1024), F.FVATTN_ERR_INVALID_ARG),       # overlapping buffers
])
def test_permute_rejects(kw, status):
    assert _permute(**kw) == status


def _route(q=FAKE, k=FAKE, p=0.9, k_min=1, ws=FAKE, ws_bytes=1 << 30, idx=FAKE, cnt=FAKE,
           hw=FAKE, grid=None, N=256, d=64):
    g = grid if grid is not None else _grid()
    return F._lib.fvattn_route(q, k, 1, 2, N, d, F.FVATTN_FP32, ctypes.byref(g), p, k_min, None,
                               None, idx, cnt, hw, ws, ws_bytes, None)


@pytest.mark.parametrize("kw, status", [
    (dict(q=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(idx=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(hw=FAKE + 4), F.FVATTN_ERR_INVALID_ARG),
    (dict(p=0.0), F.FVATTN_ERR_INVALID_ARG),
    (dict(p=1.5), F.FVATTN_ERR_INVALID_ARG),
    (dict(p=float("nan")), F.FVATTN_ERR_INVALID_ARG),
    (dict(k_min=0), F.FVATTN_ERR_INVALID_ARG),
    (dict(ws=None), F.FVATTN_ERR_WORKSPACE),
    (dict(ws=FAKE + 16), F.FVATTN_ERR_WORKSPACE),
    (dict(ws_bytes=100), F.FVATTN_ERR_WORKSPACE),
    (dict(grid=_grid(T=4096, Hh=128, W=1, th=8, tw=1), N=4096 * 128), F.FVATTN_ERR_INVALID_ARG),
])
def test_route_rejects(kw, status):
    assert _route(**kw) == status


def _sparse(qp=FAKE, op=FAKE, idx=FAKE, scale=0.125, ws=FAKE, ws_bytes=1 << 30, B=1, H=2, N=256,
            d=64, block=64, dt=F.FVATTN_FP32, blse=None):
    return F._lib.fvattn_sparse_fwd(qp, FAKE, FAKE, op, None, blse, idx, FAKE, B, H, N, d, dt, block,
                                    scale, ws, ws_bytes, None)


@pytest.mark.parametrize("kw, status", [
    (dict(qp=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(idx=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(op=FAKE + 8), F.FVATTN_ERR_INVALID_ARG),
    (dict(scale=0.0), F.FVATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), F.FVATTN_ERR_INVALID_ARG),
    (dict(d=32), F.FVATTN_ERR_INVALID_ARG),
    (dict(block=256), F.FVATTN_ERR_INVALID_ARG),
    (dict(B=0), F.FVATTN_ERR_INVALID_ARG),
    (dict(B=100, H=100), F.FVATTN_ERR_INVALID_ARG),        # B*H above the planner's limit
    (dict(ws_bytes=16), F.FVATTN_ERR_WORKSPACE),
    (dict(ws=None), F.FVATTN_ERR_WORKSPACE),
    (dict(blse=FAKE + 2), F.FVATTN_ERR_INVALID_ARG),       # block_lse must be 4-byte aligned
])
def test_sparse_rejects(kw, status):
    assert _sparse(**kw) == status


def test_dense_rejects_and_status_rejects_bad_workspace():
    assert F._lib.fvattn_dense_fwd(FAKE, FAKE, FAKE, None, None, None, 1, 1, 256, 64, F.FVATTN_FP32,
                                   64, 0.125, FAKE, 1 << 20, None) == F.FVATTN_ERR_INVALID_ARG
    assert F._lib.fvattn_workspace_status(None, None) == F.FVATTN_ERR_WORKSPACE
    assert F._lib.fvattn_workspace_status(FAKE + 64, None) == F.FVATTN_ERR_WORKSPACE


def _importance(blse=FAKE, lse=FAKE, idx=FAKE, cnt=FAKE, out=FAKE, B=1, H=2, N=256, block=64,
                ws=FAKE, ws_bytes=256):
    return F._lib.fvattn_block_importance(blse, lse, idx, cnt, B, H, N, block, out, ws, ws_bytes, None)


@pytest.mark.parametrize("kw, status", [
    (dict(blse=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(lse=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(out=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(idx=None), F.FVATTN_ERR_INVALID_ARG),           # lists given half-way
    (dict(cnt=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(lse=FAKE + 1), F.FVATTN_ERR_INVALID_ARG),
    (dict(block=96), F.FVATTN_ERR_INVALID_ARG),
    (dict(N=0), F.FVATTN_ERR_INVALID_ARG),
    (dict(ws=None), F.FVATTN_ERR_WORKSPACE),
    (dict(ws_bytes=64), F.FVATTN_ERR_WORKSPACE),
])
def test_block_importance_rejects(kw, status):
    assert _importance(**kw) == status


def _recall(imp=FAKE, idx=FAKE, cnt=FAKE, out=FAKE, B=1, H=2, N=256, block=64, ws=FAKE, ws_bytes=256):
    return F._lib.fvattn_attention_recall(imp, idx, cnt, B, H, N, block, out, ws, ws_bytes, None)


@pytest.mark.parametrize("kw, status", [
    (dict(imp=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(idx=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(cnt=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(out=FAKE + 2), F.FVATTN_ERR_INVALID_ARG),
    (dict(B=0), F.FVATTN_ERR_INVALID_ARG),
    (dict(ws=FAKE + 64), F.FVATTN_ERR_WORKSPACE),
])
def test_attention_recall_rejects(kw, status):
    assert _recall(**kw) == status


def test_diag_workspace_is_the_status_word():
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_DIAG, 1, 2, 256, 64, 64) == 256
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_DIAG, 1, 2, 256, 32, 64) == 0


def _lvsa(grid=None, B=1, H=2, window=1, period=3, step=0, idx=FAKE, cnt=FAKE, hw=FAKE, ws=FAKE,
          ws_bytes=1 << 20):
    g = grid if grid is not None else _grid()
    return F._lib.fvattn_lvsa_lists(B, H, ctypes.byref(g), window, period, step, idx, cnt, hw, ws,
                                    ws_bytes, None)


@pytest.mark.parametrize("kw, status", [
    (dict(idx=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(hw=FAKE + 4), F.FVATTN_ERR_INVALID_ARG),        # head_work must be 8-byte aligned
    (dict(window=-1), F.FVATTN_ERR_INVALID_ARG),
    (dict(period=0), F.FVATTN_ERR_INVALID_ARG),
    (dict(B=0), F.FVATTN_ERR_INVALID_ARG),
    (dict(grid=_grid(T=1100, Hh=1, W=1, th=1, tw=1)), F.FVATTN_ERR_INVALID_ARG),   # more than 1024 frames
    (dict(grid=_grid(block=32)), F.FVATTN_ERR_INVALID_ARG),
    (dict(ws=None), F.FVATTN_ERR_WORKSPACE),
    (dict(ws_bytes=256), F.FVATTN_ERR_WORKSPACE),
])
def test_lvsa_rejects(kw, status):
    assert _lvsa(**kw) == status


def test_lvsa_workspace_holds_one_frame_mask_per_block():
    nb = 4
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_LVSA, 1, 2, 256, 64, 64) == 256 + 512
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_LVSA, 1, 2, 256 * 64, 128, 64) == 256 + 256 * 128
    assert nb * 128 == 512


def test_grid_order_is_validated():
    g = _grid()
    g.order = F.FVATTN_ORDER_TABLE                      # a table order without a table
    assert F._lib.fvattn_permute(FAKE, FAKE * 4, 1, 2, 256, 64, F.FVATTN_FP32, ctypes.byref(g), 0,
                                 None) == F.FVATTN_ERR_INVALID_ARG
    g.table = FAKE + 2                                  # misaligned table
    assert F._lib.fvattn_permute(FAKE, FAKE * 4, 1, 2, 256, 64, F.FVATTN_FP32, ctypes.byref(g), 0,
                                 None) == F.FVATTN_ERR_INVALID_ARG
    g.order = 7                                         # unknown order
    assert F._lib.fvattn_permute(FAKE, FAKE * 4, 1, 2, 256, 64, F.FVATTN_FP32, ctypes.byref(g), 0,
                                 None) == F.FVATTN_ERR_INVALID_ARG
    assert ctypes.sizeof(F.Grid) == 40


def _hilbert(grid=None, table=FAKE, ws=FAKE, ws_bytes=1 << 30):
    g = grid if grid is not None else _grid()
    return F._lib.fvattn_hilbert_table(ctypes.byref(g), table, ws, ws_bytes, None)


@pytest.mark.parametrize("kw, status", [
    (dict(table=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(table=FAKE + 2), F.FVATTN_ERR_INVALID_ARG),
    (dict(grid=_grid(T=0)), F.FVATTN_ERR_INVALID_ARG),
    (dict(grid=_grid(block=96)), F.FVATTN_ERR_INVALID_ARG),
    (dict(grid=_grid(T=4097, Hh=1, W=128)), F.FVATTN_ERR_INVALID_ARG),          # more than 4096 blocks
    (dict(grid=_grid(T=1, Hh=1, W=1 << 19, block=128)), F.FVATTN_ERR_UNSUPPORTED),  # 3*19 + 19 key bits
    (dict(ws=None), F.FVATTN_ERR_WORKSPACE),
    (dict(ws_bytes=1024), F.FVATTN_ERR_WORKSPACE),
])
def test_hilbert_table_rejects(kw, status):
    assert _hilbert(**kw) == status


def test_hilbert_workspace_holds_the_padded_keys():
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_HILBERT, 1, 1, 75600, 64, 128) == 256 + (1 << 17) * 8


def test_empty_inputs_are_rejected_before_any_launch():
    # N = 0 tokens (an empty grid) at every entry point that takes N
    g0 = _grid(T=0)
    assert F._lib.fvattn_permute(FAKE, FAKE * 4, 1, 2, 0, 64, F.FVATTN_FP32, ctypes.byref(g0), 0,
                                 None) == F.FVATTN_ERR_INVALID_ARG
    assert _route(grid=g0, N=0) == F.FVATTN_ERR_INVALID_ARG
    assert _sparse(N=0) == F.FVATTN_ERR_INVALID_ARG
    assert F._lib.fvattn_dense_fwd(FAKE, FAKE, FAKE, FAKE, None, None, 1, 2, 0, 64, F.FVATTN_FP32, 64,
                                   0.125, FAKE, 1 << 20, None) == F.FVATTN_ERR_INVALID_ARG
    assert _lvsa(grid=g0) == F.FVATTN_ERR_INVALID_ARG
    assert _hilbert(grid=g0) == F.FVATTN_ERR_INVALID_ARG
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_SPARSE_FWD, 1, 2, 0, 64, 64) == 0


def _select(imp=FAKE, idx=FAKE, cnt=FAKE, hw=FAKE, p=0.8, k_min=1, B=1, H=2, N=256, block=64, ws=FAKE,
            ws_bytes=256):
    return F._lib.fvattn_select_topp(imp, B, H, N, block, p, k_min, idx, cnt, hw, ws, ws_bytes, None)


@pytest.mark.parametrize("kw, status", [
    (dict(imp=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(hw=FAKE + 4), F.FVATTN_ERR_INVALID_ARG),
    (dict(p=0.0), F.FVATTN_ERR_INVALID_ARG),
    (dict(p=1.5), F.FVATTN_ERR_INVALID_ARG),
    (dict(k_min=0), F.FVATTN_ERR_INVALID_ARG),
    (dict(N=0), F.FVATTN_ERR_INVALID_ARG),
    (dict(ws=None), F.FVATTN_ERR_WORKSPACE),
])
def test_select_topp_rejects(kw, status):
    assert _select(**kw) == status


def _quant(vp=FAKE, vq=FAKE + (1 << 24), vs=FAKE + (1 << 26), B=1, H=2, N=256, d=128, block=64, ws=FAKE + (1 << 28),
           ws_bytes=1 << 20):
    return F._lib.fvattn_quantize_v(vp, B, H, N, d, block, vq, vs, ws, ws_bytes, None)


@pytest.mark.parametrize("kw, status", [
    (dict(vp=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(vq=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(vs=FAKE + (1 << 26) + 4), F.FVATTN_ERR_INVALID_ARG),
    (dict(vq=FAKE + 4096), F.FVATTN_ERR_INVALID_ARG),            # overlaps vp
    (dict(N=0), F.FVATTN_ERR_INVALID_ARG),
    (dict(block=96), F.FVATTN_ERR_INVALID_ARG),
    (dict(d=64), F.FVATTN_ERR_UNSUPPORTED),
    (dict(ws=None), F.FVATTN_ERR_WORKSPACE),
    (dict(ws_bytes=16), F.FVATTN_ERR_WORKSPACE),
])
def test_quantize_v_rejects(kw, status):
    assert _quant(**kw) == status


def test_quantize_v_workspace_holds_channel_maxima():
    hdr = F.fvattn_workspace_bytes(F.FVATTN_OP_DENSE_FWD, 1, 1, 256, 128, 64)
    assert F.fvattn_workspace_bytes(F.FVATTN_OP_QUANT_V, 2, 3, 256, 128, 64) >= hdr + 6 * 128 * 4


def _fp8(sparse=True, vq=FAKE, vs=FAKE, d=128, idx=FAKE, scale=0.125, ws=FAKE, ws_bytes=1 << 30):
    if sparse:
        return F._lib.fvattn_sparse_fwd_fp8v(FAKE, FAKE, vq, vs, FAKE, None, None, idx, FAKE, 1, 2, 256, d, 64,
                                             scale, ws, ws_bytes, None)
    return F._lib.fvattn_dense_fwd_fp8v(FAKE, FAKE, vq, vs, FAKE, None, None, 1, 2, 256, d, 64, scale, ws,
                                        ws_bytes, None)


@pytest.mark.parametrize("sparse", [True, False])
@pytest.mark.parametrize("kw, status", [
    (dict(vs=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(vs=FAKE + 4), F.FVATTN_ERR_INVALID_ARG),
    (dict(vq=None), F.FVATTN_ERR_INVALID_ARG),
    (dict(scale=0.0), F.FVATTN_ERR_INVALID_ARG),
    (dict(d=64), F.FVATTN_ERR_UNSUPPORTED),
    (dict(ws=None), F.FVATTN_ERR_WORKSPACE),
])
def test_fp8v_attention_rejects(sparse, kw, status):
    assert _fp8(sparse=sparse, **kw) == status


def test_sparse_fp8v_rejects_missing_lists():
    assert _fp8(idx=None) == F.FVATTN_ERR_INVALID_ARG
