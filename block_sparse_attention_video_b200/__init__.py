"""Python binding of libfvattn.so (include/fvattn.h): argument marshalling only.

Every step of the attention path runs in the library's CUDA kernels; this
module turns torch tensors into pointers and sizes, passes the current CUDA
stream, and raises on a non-OK status. It never computes on the CPU and has no
fallback: importing it fails loudly if the library has not been built
(``python block_sparse_attention_video_b200/build_lib.py``).

Entry points carry the C names: ``fvattn_permute``, ``fvattn_route``,
``fvattn_route_noalloc``, ``fvattn_sparse_fwd``, ``fvattn_dense_fwd``,
``fvattn_block_importance``, ``fvattn_attention_recall``, ``fvattn_select_topp``, ``fvattn_lvsa_lists``,
``fvattn_hilbert_table``, ``fvattn_quantize_v``, ``fvattn_sparse_fwd_fp8v``, ``fvattn_dense_fwd_fp8v``,
``fvattn_workspace_bytes``, ``fvattn_workspace_status``, ``fvattn_wait_selftest``. ``FVAttnPath`` strings
them into the full per-call
path (route -> permute V -> block-sparse attention -> inverse permute) over
buffers it allocates once with torch; ``HostPipeline`` runs it over a sequence
of calls with pinned host inputs and outputs, overlapping the copies of
neighbouring calls with the kernels of the current one.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfvattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python block_sparse_attention_video_b200/build_lib.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

FVATTN_OK = 0
FVATTN_ERR_INVALID_ARG = 1
FVATTN_ERR_UNSUPPORTED = 2
FVATTN_ERR_WORKSPACE = 3
FVATTN_ERR_CUDA = 4
FVATTN_ERR_TIMEOUT = 5

FVATTN_BF16 = 0
FVATTN_FP32 = 1

FVATTN_OP_ROUTE = 0
FVATTN_OP_SPARSE_FWD = 1
FVATTN_OP_DENSE_FWD = 2
FVATTN_OP_DIAG = 3
FVATTN_OP_LVSA = 4
FVATTN_OP_HILBERT = 5
FVATTN_OP_QUANT_V = 6

FVATTN_ORDER_TILES = 0
FVATTN_ORDER_TABLE = 1

EXPORTED = ("fvattn_workspace_bytes", "fvattn_permute", "fvattn_route", "fvattn_route_noalloc",
            "fvattn_sparse_fwd", "fvattn_dense_fwd", "fvattn_block_importance", "fvattn_attention_recall",
            "fvattn_select_topp", "fvattn_lvsa_lists", "fvattn_hilbert_table", "fvattn_quantize_v",
            "fvattn_sparse_fwd_fp8v", "fvattn_dense_fwd_fp8v",
            "fvattn_workspace_status", "fvattn_status_string", "fvattn_wait_selftest",
            "fvattn_permute_quantize_v", "fvattn_order_lists_by_importance")


class Grid(ctypes.Structure):
    """fvattn_grid: latent video grid (T, Hh, W), tiles (tt, th, tw), block size, and
    block order (3-D tiles, or an explicit device table such as the Hilbert order)."""
    _fields_ = [("T", ctypes.c_int), ("Hh", ctypes.c_int), ("W", ctypes.c_int),
                ("tt", ctypes.c_int), ("th", ctypes.c_int), ("tw", ctypes.c_int),
                ("block", ctypes.c_int), ("order", ctypes.c_int), ("table", ctypes.c_void_p)]

    @classmethod
    def make(cls, grid, tile, block, table=None):
        """Tile order, or the explicit order of ``table`` (an int32 CUDA tensor [N])."""
        g = cls(*grid, *tile, block, FVATTN_ORDER_TILES if table is None else FVATTN_ORDER_TABLE,
                None if table is None else table.data_ptr())
        g._table = table          # keeps the table's storage alive with the grid
        return g

    @property
    def N(self):
        return self.T * self.Hh * self.W

    @property
    def nb(self):
        return -(-self.N // self.block)


_c_int, _c_void_p, _c_float, _c_size_t = ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
_lib.fvattn_workspace_bytes.argtypes = [_c_int] * 6
_lib.fvattn_workspace_bytes.restype = _c_size_t
_lib.fvattn_permute.argtypes = [_c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                                ctypes.POINTER(Grid), _c_int, _c_void_p]
_lib.fvattn_permute.restype = _c_int
_lib.fvattn_route.argtypes = [_c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                              ctypes.POINTER(Grid), _c_float, _c_int, _c_void_p, _c_void_p,
                              _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_route.restype = _c_int
_lib.fvattn_route_noalloc.argtypes = [_c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                                      ctypes.POINTER(Grid), _c_float, _c_int, _c_void_p, _c_void_p,
                                      _c_void_p, _c_void_p, _c_void_p, _c_void_p]
_lib.fvattn_route_noalloc.restype = _c_int
_lib.fvattn_order_lists_by_importance.argtypes = [_c_void_p, _c_void_p] + [_c_int] * 5 + [_c_void_p, _c_size_t,
                                                                                       _c_void_p]
_lib.fvattn_order_lists_by_importance.restype = _c_int
_lib.fvattn_sparse_fwd.argtypes = [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                   _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int,
                                   _c_int, _c_int, _c_float, _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_sparse_fwd.restype = _c_int
_lib.fvattn_dense_fwd.argtypes = [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                  _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                                  _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_dense_fwd.restype = _c_int
_lib.fvattn_quantize_v.argtypes = [_c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_void_p, _c_void_p,
                                   _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_quantize_v.restype = _c_int
_lib.fvattn_permute_quantize_v.argtypes = [_c_void_p, _c_int, _c_int, _c_int, _c_int, ctypes.POINTER(Grid),
                                           _c_void_p, _c_void_p, _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_permute_quantize_v.restype = _c_int
_lib.fvattn_sparse_fwd_fp8v.argtypes = [_c_void_p] * 9 + [_c_int] * 5 + [_c_float, _c_void_p, _c_size_t,
                                                                      _c_void_p]
_lib.fvattn_sparse_fwd_fp8v.restype = _c_int
_lib.fvattn_dense_fwd_fp8v.argtypes = [_c_void_p] * 7 + [_c_int] * 5 + [_c_float, _c_void_p, _c_size_t,
                                                                     _c_void_p]
_lib.fvattn_dense_fwd_fp8v.restype = _c_int
_lib.fvattn_block_importance.argtypes = [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int,
                                         _c_int, _c_int, _c_void_p, _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_block_importance.restype = _c_int
_lib.fvattn_attention_recall.argtypes = [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int,
                                         _c_int, _c_void_p, _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_attention_recall.restype = _c_int
_lib.fvattn_select_topp.argtypes = [_c_void_p, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_void_p,
                                    _c_void_p, _c_void_p, _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_select_topp.restype = _c_int
_lib.fvattn_lvsa_lists.argtypes = [_c_int, _c_int, ctypes.POINTER(Grid), _c_int, _c_int, _c_int, _c_void_p,
                                   _c_void_p, _c_void_p, _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_lvsa_lists.restype = _c_int
_lib.fvattn_hilbert_table.argtypes = [ctypes.POINTER(Grid), _c_void_p, _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_hilbert_table.restype = _c_int
_lib.fvattn_workspace_status.argtypes = [_c_void_p, _c_void_p]
_lib.fvattn_workspace_status.restype = _c_int
_lib.fvattn_wait_selftest.argtypes = [_c_void_p, _c_void_p, _c_size_t, _c_void_p]
_lib.fvattn_wait_selftest.restype = _c_int
_lib.fvattn_status_string.argtypes = [_c_int]
_lib.fvattn_status_string.restype = ctypes.c_char_p


class FVAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fvattn_status_string(status)} (status {status})")


def fvattn_status_string(status: int) -> str:
    return _lib.fvattn_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != FVATTN_OK:
        raise FVAttnError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None):
    """The given stream (which must belong to ``device``), else ``device``'s current stream."""
    if stream is None:
        s = torch.cuda.current_stream(device)
    else:
        s = stream
        if device is not None and s.device != torch.device(device):
            raise ValueError(f"stream is on {s.device}, tensors on {device}")
    return ctypes.c_void_p(s.cuda_stream)


def _expect(t, name, dev, shape=None, dtype=None, optional=False):
    """Every buffer handed to the library: a contiguous CUDA tensor on ``dev`` with the
    shape and dtype the C call assumes (the library sees only a pointer, so a wrong size
    would make a kernel read or write past the end of the buffer)."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device != dev:
        raise ValueError(f"{name} is on {t.device}, expected {dev}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _expect_ws(ws, dev):
    _expect(ws, "workspace", dev)


def _call(dev, fn, *args):
    """Runs a library call with ``dev`` current, so that device-side lookups (SM count,
    static scratch) and launches happen on the tensors' device."""
    with torch.cuda.device(dev):
        return fn(*args)


def _nb(N, block):
    return -(-int(N) // int(block))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FVATTN_BF16
    if t.dtype == torch.float32:
        return FVATTN_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def fvattn_workspace_bytes(op: int, B: int, H: int, N: int, d: int, block: int) -> int:
    return int(_lib.fvattn_workspace_bytes(op, B, H, N, d, block))


def fvattn_permute(x, y, grid: Grid, inverse: bool = False, stream=None):
    """x [B,H,N,d] -> y [B,H,Npad,d] (tile order), or the inverse."""
    _need_cuda(x, y)
    dev = x.device
    B, H, n_in, d = x.shape
    npad = grid.nb * grid.block
    if n_in != (npad if inverse else grid.N):
        raise ValueError(f"x has {n_in} rows, expected {npad if inverse else grid.N}")
    _expect(y, "y", dev, (B, H, grid.N if inverse else npad, d), x.dtype)
    _check(_call(dev, _lib.fvattn_permute, _ptr(x), _ptr(y), B, H, grid.N, d, _dtype_code(x),
                 ctypes.byref(grid), 1 if inverse else 0, _stream(stream, dev)), "fvattn_permute")
    return y


def fvattn_route(q, k, grid: Grid, p: float, k_min: int, kv_idx, kv_cnt, head_work, workspace,
                 qp_out=None, kp_out=None, stream=None):
    """Routing front end; fills kv_idx [B,H,nb,nb], kv_cnt [B,H,nb], head_work [B,H]."""
    _need_cuda(q, k, kv_idx, kv_cnt, head_work, workspace, qp_out, kp_out)
    dev = q.device
    B, H, N, d = q.shape
    _check_route_buffers(q, k, grid, kv_idx, kv_cnt, head_work, qp_out, kp_out)
    _expect_ws(workspace, dev)
    _check(_call(dev, _lib.fvattn_route, _ptr(q), _ptr(k), B, H, N, d, _dtype_code(q), ctypes.byref(grid),
                 float(p), int(k_min), _ptr(qp_out), _ptr(kp_out), _ptr(kv_idx),
                 _ptr(kv_cnt), _ptr(head_work), _ptr(workspace),
                 workspace.numel() * workspace.element_size(), _stream(stream, dev)),
           "fvattn_route")
    return kv_idx, kv_cnt, head_work


def _check_lists(kv_idx, kv_cnt, head_work, dev, B, H, nb):
    _expect(kv_idx, "kv_idx", dev, (B, H, nb, nb), torch.int32)
    _expect(kv_cnt, "kv_cnt", dev, (B, H, nb), torch.int32)
    _expect(head_work, "head_work", dev, (B, H), torch.int64, optional=head_work is None)


def _check_route_buffers(q, k, grid, kv_idx, kv_cnt, head_work, qp_out, kp_out):
    dev = q.device
    B, H, N, d = q.shape
    if N != grid.N:
        raise ValueError(f"q has {N} tokens, the grid {grid.N}")
    _dtype_code(q)
    _expect(k, "k", dev, q.shape, q.dtype)
    nb = grid.nb
    _check_lists(kv_idx, kv_cnt, head_work, dev, B, H, nb)
    for t, name in ((qp_out, "qp_out"), (kp_out, "kp_out")):
        _expect(t, name, dev, (B, H, nb * grid.block, d), q.dtype, optional=True)


def fvattn_order_lists_by_importance(kv_idx, kv_cnt, N: int, d: int, block: int, workspace, stream=None):
    """Reorders the lists of the preceding fvattn_route call made with this workspace
    by descending block score (ties by block index), in place."""
    _need_cuda(kv_idx, kv_cnt, workspace)
    dev = kv_cnt.device
    B, H, nb = kv_cnt.shape
    if nb != _nb(N, block):
        raise ValueError(f"kv_cnt has {nb} blocks per row, expected {_nb(N, block)}")
    _check_lists(kv_idx, kv_cnt, None, dev, B, H, nb)
    _expect_ws(workspace, dev)
    _check(_call(dev, _lib.fvattn_order_lists_by_importance, _ptr(kv_idx), _ptr(kv_cnt), B, H, N, d, block,
                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream, dev)),
           "fvattn_order_lists_by_importance")
    return kv_idx


def fvattn_route_noalloc(q, k, grid: Grid, p: float, k_min: int, kv_idx, kv_cnt, head_work,
                         qp_out=None, kp_out=None, stream=None):
    """fvattn_route without a workspace, for callers that cannot allocate device
    memory where they route; the library's static 96 MiB device scratch is used
    instead (calls that overlap on the GPU race on it)."""
    _need_cuda(q, k, kv_idx, kv_cnt, head_work, qp_out, kp_out)
    dev = q.device
    B, H, N, d = q.shape
    _check_route_buffers(q, k, grid, kv_idx, kv_cnt, head_work, qp_out, kp_out)
    _check(_call(dev, _lib.fvattn_route_noalloc, _ptr(q), _ptr(k), B, H, N, d, _dtype_code(q),
                 ctypes.byref(grid), float(p), int(k_min), _ptr(qp_out), _ptr(kp_out), _ptr(kv_idx),
                 _ptr(kv_cnt), _ptr(head_work), _stream(stream, dev)),
           "fvattn_route_noalloc")
    return kv_idx, kv_cnt, head_work


def _check_attn(qp, kp, v, out, N, block, workspace, lse, block_lse, v_dtype=None, vscale=None):
    """Shapes of an attention call: qp, kp, out [B,H,Npad,d] of one dtype; v the same
    shape (bf16/fp32 like qp, or E4M3 codes as uint8 with vscale [B,H,d] fp32);
    lse [B,H,Npad] and block_lse [B,H,nb,Npad] fp32 when given."""
    dev = qp.device
    B, H, npad, d = qp.shape
    nb = _nb(N, block)
    if npad != nb * block:
        raise ValueError(f"qp has {npad} rows, expected {nb * block} (N={N}, block={block})")
    _dtype_code(qp)
    _expect(kp, "kp", dev, qp.shape, qp.dtype)
    _expect(v, "v", dev, qp.shape, v_dtype or qp.dtype)
    _expect(out, "out", dev, qp.shape, qp.dtype)
    _expect(vscale, "vscale", dev, (B, H, d), torch.float32, optional=vscale is None)
    _expect(lse, "lse", dev, (B, H, npad), torch.float32, optional=True)
    _expect(block_lse, "block_lse", dev, (B, H, nb, npad), torch.float32, optional=True)
    _expect_ws(workspace, dev)
    return dev, B, H, d, nb


def fvattn_sparse_fwd(qp, kp, vp, out, kv_idx, kv_cnt, N: int, block: int, workspace,
                      scale=None, lse=None, block_lse=None, stream=None):
    """Block-sparse attention over permuted [B,H,Npad,d] tensors; optional lse
    [B,H,Npad] and block_lse [B,H,nb,Npad] (fp32) outputs."""
    _need_cuda(qp, kp, vp, out, kv_idx, kv_cnt, workspace, lse, block_lse)
    dev, B, H, d, nb = _check_attn(qp, kp, vp, out, N, block, workspace, lse, block_lse)
    _check_lists(kv_idx, kv_cnt, None, dev, B, H, nb)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(_call(dev, _lib.fvattn_sparse_fwd, _ptr(qp), _ptr(kp), _ptr(vp), _ptr(out), _ptr(lse),
                 _ptr(block_lse), _ptr(kv_idx), _ptr(kv_cnt), B, H, N, d, _dtype_code(qp), block, sc,
                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                 _stream(stream, dev)), "fvattn_sparse_fwd")
    return out


def fvattn_dense_fwd(qp, kp, vp, out, N: int, block: int, workspace, scale=None, lse=None,
                     block_lse=None, stream=None):
    """Dense attention over permuted [B,H,Npad,d] tensors (every key block)."""
    _need_cuda(qp, kp, vp, out, workspace, lse, block_lse)
    dev, B, H, d, nb = _check_attn(qp, kp, vp, out, N, block, workspace, lse, block_lse)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(_call(dev, _lib.fvattn_dense_fwd, _ptr(qp), _ptr(kp), _ptr(vp), _ptr(out), _ptr(lse),
                 _ptr(block_lse), B, H, N, d, _dtype_code(qp), block, sc, _ptr(workspace),
                 workspace.numel() * workspace.element_size(), _stream(stream, dev)),
           "fvattn_dense_fwd")
    return out


def fvattn_quantize_v(vp, vq, vscale, N: int, block: int, workspace, stream=None):
    """Per-channel E4M3 quantization: vp [B,H,Npad,128] bf16 -> vq [B,H,Npad,128]
    uint8 codes and vscale [B,H,128] fp32."""
    _need_cuda(vp, vq, vscale, workspace)
    dev = vp.device
    B, H, npad, d = vp.shape
    if vp.dtype != torch.bfloat16 or vq.dtype != torch.uint8 or vscale.dtype != torch.float32:
        raise TypeError("vp bf16, vq uint8, vscale float32")
    if npad != _nb(N, block) * block:
        raise ValueError(f"vp has {npad} rows, expected {_nb(N, block) * block}")
    _expect(vq, "vq", dev, vp.shape, torch.uint8)
    _expect(vscale, "vscale", dev, (B, H, d), torch.float32)
    _expect_ws(workspace, dev)
    _check(_call(dev, _lib.fvattn_quantize_v, _ptr(vp), B, H, N, d, block, _ptr(vq), _ptr(vscale),
                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream, dev)),
           "fvattn_quantize_v")
    return vq, vscale


def fvattn_permute_quantize_v(v, grid: Grid, vq, vscale, workspace, stream=None):
    """Raster-order V [B,H,N,128] bf16 -> E4M3 codes vq [B,H,Npad,128] uint8 in the grid's
    block order and scales vscale [B,H,128] fp32 (the permutation and the quantization
    in one pass over the codes)."""
    _need_cuda(v, vq, vscale, workspace)
    dev = v.device
    B, H, N, d = v.shape
    if v.dtype != torch.bfloat16:
        raise TypeError("v must be bf16")
    if N != grid.N:
        raise ValueError(f"v has {N} tokens, the grid {grid.N}")
    _expect(vq, "vq", dev, (B, H, grid.nb * grid.block, d), torch.uint8)
    _expect(vscale, "vscale", dev, (B, H, d), torch.float32)
    _expect_ws(workspace, dev)
    _check(_call(dev, _lib.fvattn_permute_quantize_v, _ptr(v), B, H, N, d, ctypes.byref(grid), _ptr(vq),
                 _ptr(vscale), _ptr(workspace), workspace.numel() * workspace.element_size(),
                 _stream(stream, dev)), "fvattn_permute_quantize_v")
    return vq, vscale


def fvattn_sparse_fwd_fp8v(qp, kp, vq, vscale, out, kv_idx, kv_cnt, N: int, block: int, workspace,
                           scale=None, lse=None, block_lse=None, stream=None):
    """fvattn_sparse_fwd with the E4M3 V of fvattn_quantize_v (8-bit P.V product)."""
    _need_cuda(qp, kp, vq, vscale, out, kv_idx, kv_cnt, workspace, lse, block_lse)
    dev, B, H, d, nb = _check_attn(qp, kp, vq, out, N, block, workspace, lse, block_lse,
                                   v_dtype=torch.uint8, vscale=vscale)
    _check_lists(kv_idx, kv_cnt, None, dev, B, H, nb)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(_call(dev, _lib.fvattn_sparse_fwd_fp8v, _ptr(qp), _ptr(kp), _ptr(vq), _ptr(vscale), _ptr(out),
                 _ptr(lse), _ptr(block_lse), _ptr(kv_idx), _ptr(kv_cnt), B, H, N, d, block, sc,
                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                 _stream(stream, dev)), "fvattn_sparse_fwd_fp8v")
    return out


def fvattn_dense_fwd_fp8v(qp, kp, vq, vscale, out, N: int, block: int, workspace, scale=None, lse=None,
                          block_lse=None, stream=None):
    """fvattn_dense_fwd with the E4M3 V of fvattn_quantize_v (8-bit P.V product)."""
    _need_cuda(qp, kp, vq, vscale, out, workspace, lse, block_lse)
    dev, B, H, d, nb = _check_attn(qp, kp, vq, out, N, block, workspace, lse, block_lse,
                                   v_dtype=torch.uint8, vscale=vscale)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(_call(dev, _lib.fvattn_dense_fwd_fp8v, _ptr(qp), _ptr(kp), _ptr(vq), _ptr(vscale), _ptr(out),
                 _ptr(lse), _ptr(block_lse), B, H, N, d, block, sc, _ptr(workspace),
                 workspace.numel() * workspace.element_size(), _stream(stream, dev)),
           "fvattn_dense_fwd_fp8v")
    return out


def fvattn_block_importance(block_lse, lse, importance, N: int, block: int, workspace,
                            kv_idx=None, kv_cnt=None, stream=None):
    """Exact block importance [B,H,nb,nb] from an attention call's block_lse and lse
    (kv_idx/kv_cnt: the call's lists; None for a dense call)."""
    _need_cuda(block_lse, lse, importance, workspace, kv_idx, kv_cnt)
    dev = lse.device
    B, H = lse.shape[:2]
    nb = _nb(N, block)
    npad = nb * block
    _expect(lse, "lse", dev, (B, H, npad), torch.float32)
    _expect(block_lse, "block_lse", dev, (B, H, nb, npad), torch.float32)
    _expect(importance, "importance", dev, (B, H, nb, nb), torch.float32)
    if (kv_idx is None) != (kv_cnt is None):
        raise ValueError("kv_idx and kv_cnt go together")
    if kv_idx is not None:
        _check_lists(kv_idx, kv_cnt, None, dev, B, H, nb)
    _expect_ws(workspace, dev)
    _check(_call(dev, _lib.fvattn_block_importance, _ptr(block_lse), _ptr(lse), _ptr(kv_idx), _ptr(kv_cnt),
                 B, H, N, block, _ptr(importance), _ptr(workspace),
                 workspace.numel() * workspace.element_size(), _stream(stream, dev)),
           "fvattn_block_importance")
    return importance


def fvattn_attention_recall(importance, kv_idx, kv_cnt, recall, N: int, block: int, workspace,
                            stream=None):
    """Per query block, the dense importance captured by the lists: recall [B,H,nb]."""
    _need_cuda(importance, kv_idx, kv_cnt, recall, workspace)
    dev = kv_cnt.device
    B, H = kv_cnt.shape[:2]
    nb = _nb(N, block)
    _check_lists(kv_idx, kv_cnt, None, dev, B, H, nb)
    _expect(importance, "importance", dev, (B, H, nb, nb), torch.float32)
    _expect(recall, "recall", dev, (B, H, nb), torch.float32)
    _expect_ws(workspace, dev)
    _check(_call(dev, _lib.fvattn_attention_recall, _ptr(importance), _ptr(kv_idx), _ptr(kv_cnt), B, H, N,
                 block, _ptr(recall), _ptr(workspace), workspace.numel() * workspace.element_size(),
                 _stream(stream, dev)),
           "fvattn_attention_recall")
    return recall


def fvattn_select_topp(importance, N: int, block: int, p: float, k_min: int, kv_idx, kv_cnt, head_work,
                       workspace, stream=None):
    """Top-p + Top-k floor on importance rows [B,H,nb,nb] (the GSRS search over a candidate set)."""
    _need_cuda(importance, kv_idx, kv_cnt, head_work, workspace)
    dev = kv_cnt.device
    B, H = kv_cnt.shape[:2]
    nb = _nb(N, block)
    _check_lists(kv_idx, kv_cnt, head_work, dev, B, H, nb)
    _expect(importance, "importance", dev, (B, H, nb, nb), torch.float32)
    _expect_ws(workspace, dev)
    _check(_call(dev, _lib.fvattn_select_topp, _ptr(importance), B, H, N, block, float(p), int(k_min),
                 _ptr(kv_idx), _ptr(kv_cnt), _ptr(head_work), _ptr(workspace),
                 workspace.numel() * workspace.element_size(), _stream(stream, dev)),
           "fvattn_select_topp")
    return kv_idx, kv_cnt, head_work


def fvattn_lvsa_lists(grid: Grid, window: int, period: int, step: int, kv_idx, kv_cnt, head_work,
                      workspace, stream=None):
    """LVSA window + rotating global-frame lists for every (b, h) of kv_cnt's [B,H,nb] shape."""
    _need_cuda(kv_idx, kv_cnt, head_work, workspace)
    dev = kv_cnt.device
    B, H = kv_cnt.shape[:2]
    _check_lists(kv_idx, kv_cnt, head_work, dev, B, H, grid.nb)
    _expect_ws(workspace, dev)
    _check(_call(dev, _lib.fvattn_lvsa_lists, B, H, ctypes.byref(grid), int(window), int(period), int(step),
                 _ptr(kv_idx), _ptr(kv_cnt), _ptr(head_work), _ptr(workspace),
                 workspace.numel() * workspace.element_size(), _stream(stream, dev)),
           "fvattn_lvsa_lists")
    return kv_idx, kv_cnt, head_work


def fvattn_hilbert_table(grid_thw, block: int = 128, device="cuda", stream=None) -> torch.Tensor:
    """Hilbert-curve order of grid (T, Hh, W): int32 [N] with table[pos] = raster index."""
    T, Hh, W = grid_thw
    g = Grid(T, Hh, W, 1, 1, 1, block, FVATTN_ORDER_TILES, None)
    N = T * Hh * W
    table = torch.empty(N, dtype=torch.int32, device=device)
    dev = table.device
    ws = alloc_workspace(fvattn_workspace_bytes(FVATTN_OP_HILBERT, 1, 1, N, 64, block), dev)
    _check(_call(dev, _lib.fvattn_hilbert_table, ctypes.byref(g), _ptr(table), _ptr(ws),
                 ws.numel() * ws.element_size(), _stream(stream, dev)),
           "fvattn_hilbert_table")
    torch.cuda.current_stream(dev).synchronize() if stream is None else stream.synchronize()
    return table


def fvattn_workspace_status(workspace, stream=None) -> int:
    """Synchronize the stream and return the status word the kernels recorded."""
    _need_cuda(workspace)
    dev = workspace.device
    return int(_call(dev, _lib.fvattn_workspace_status, _ptr(workspace), _stream(stream, dev)))


def fvattn_wait_selftest(results, workspace, stream=None):
    """Runs the bounded-wait self-test (no fault: waits on barriers nothing arrives at);
    results [8] int64 on the device. The status word then reads FVATTN_ERR_TIMEOUT."""
    _need_cuda(results, workspace)
    dev = results.device
    _expect(results, "results", dev, (8,), torch.int64)
    _expect_ws(workspace, dev)
    _check(_call(dev, _lib.fvattn_wait_selftest, _ptr(results), _ptr(workspace),
                 workspace.numel() * workspace.element_size(), _stream(stream, dev)), "fvattn_wait_selftest")
    return results


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned uint8 buffer (torch's caching allocator aligns to 512)."""
    t = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    assert t.data_ptr() % 256 == 0
    return t


class FVAttnPath:
    """The whole per-call path on one device with buffers allocated once.

    ``__call__(q, k, v)`` takes [B,H,N,d] tensors in original token order and
    returns the attention output [B,H,N,d] in original order: route (which
    also permutes q and k), permute v, block-sparse attention, inverse permute.
    ``dense=True`` runs the dense kernel instead of routing. ``order="hilbert"``
    orders blocks along the Hilbert curve (the table is built once here) instead
    of 3-D tiles. ``v_format="e4m3"`` permutes and quantizes V per channel in one
    call (fvattn_permute_quantize_v; no bf16 permuted V is formed) and runs
    attention with the 8-bit P.V product.
    """

    def __init__(self, B, H, grid, tile, block, d, dtype, p, k_min, device="cuda", order="tiles",
                 v_format="bf16", _grid=None):
        if order not in ("tiles", "hilbert"):
            raise ValueError(f"unknown block order {order!r}")
        if v_format not in ("bf16", "e4m3"):
            raise ValueError(f"unknown V format {v_format!r}")
        self.fp8v = v_format == "e4m3"
        self._ctor = dict(grid=grid, tile=tile, block=block, d=d, dtype=dtype, p=p, k_min=k_min, device=device,
                          order=order, v_format=v_format)
        if _grid is not None:
            self.grid = _grid                 # shared with the path it was split from
        else:
            table = fvattn_hilbert_table(grid, block, device) if order == "hilbert" else None
            self.grid = Grid.make(grid, tile, block, table=table)
        self.B, self.H, self.d = B, H, d
        self.N, self.nb = self.grid.N, self.grid.nb
        self.npad = self.nb * block
        self.block = block
        self.p, self.k_min = float(p), int(k_min)
        self.dtype = dtype
        dev = torch.device(device)
        shp = (B, H, self.npad, d)
        self.qp = torch.empty(shp, dtype=dtype, device=dev)
        self.kp = torch.empty(shp, dtype=dtype, device=dev)
        self.vp = None if self.fp8v else torch.empty(shp, dtype=dtype, device=dev)
        self.op = torch.empty(shp, dtype=dtype, device=dev)
        self.out = torch.empty((B, H, self.N, d), dtype=dtype, device=dev)
        self.kv_idx = torch.empty((B, H, self.nb, self.nb), dtype=torch.int32, device=dev)
        self.kv_cnt = torch.empty((B, H, self.nb), dtype=torch.int32, device=dev)
        self.head_work = torch.empty((B, H), dtype=torch.int64, device=dev)
        self.ws_route = alloc_workspace(
            fvattn_workspace_bytes(FVATTN_OP_ROUTE, B, H, self.N, d, block), dev)
        self.ws_attn = alloc_workspace(
            fvattn_workspace_bytes(FVATTN_OP_SPARSE_FWD, B, H, self.N, d, block), dev)
        if self.fp8v:
            self.vq = torch.empty(shp, dtype=torch.uint8, device=dev)
            self.vscale = torch.empty((B, H, d), dtype=torch.float32, device=dev)
            self.ws_quant = alloc_workspace(
                fvattn_workspace_bytes(FVATTN_OP_QUANT_V, B, H, self.N, d, block), dev)

    def split_heads(self, groups):
        """Paths over contiguous head ranges (B must be 1), each with its own buffers and
        workspaces, sharing this path's grid (and Hilbert table). Heads are independent,
        so running the sub-paths on head slices gives exactly this path's result.
        Returns [(h0, h1, path)]."""
        if self.B != 1:
            raise ValueError("head groups need B == 1 (a head range is then contiguous)")
        groups = max(1, min(int(groups), self.H))
        bounds = [round(g * self.H / groups) for g in range(groups + 1)]
        out = []
        for h0, h1 in zip(bounds[:-1], bounds[1:]):
            c = self._ctor
            sub = FVAttnPath(1, h1 - h0, c["grid"], c["tile"], c["block"], c["d"], c["dtype"], self.p, self.k_min,
                             device=c["device"], order=c["order"], v_format=c["v_format"], _grid=self.grid)
            out.append((h0, h1, sub))
        return out

    def route(self, q, k):
        fvattn_route(q, k, self.grid, self.p, self.k_min, self.kv_idx, self.kv_cnt,
                     self.head_work, self.ws_route, qp_out=self.qp, kp_out=self.kp)

    def prepare_v(self, v):
        """V [B,H,N,d] (original order) into the attention kernel's input: the permuted
        bf16 V, or (E4M3 path) the permuted per-channel E4M3 codes and scales, formed
        from the raster-order V in one fused call."""
        if self.fp8v:
            fvattn_permute_quantize_v(v, self.grid, self.vq, self.vscale, self.ws_quant)
        else:
            fvattn_permute(v, self.vp, self.grid)

    def attend(self, dense=False):
        """Attention over the prepared inputs (qp, kp from route or permute; V from
        prepare_v)."""
        if self.fp8v:
            if dense:
                fvattn_dense_fwd_fp8v(self.qp, self.kp, self.vq, self.vscale, self.op, self.N, self.block,
                                      self.ws_attn)
            else:
                fvattn_sparse_fwd_fp8v(self.qp, self.kp, self.vq, self.vscale, self.op, self.kv_idx,
                                       self.kv_cnt, self.N, self.block, self.ws_attn)
        elif dense:
            fvattn_dense_fwd(self.qp, self.kp, self.vp, self.op, self.N, self.block, self.ws_attn)
        else:
            fvattn_sparse_fwd(self.qp, self.kp, self.vp, self.op, self.kv_idx, self.kv_cnt,
                              self.N, self.block, self.ws_attn)

    def __call__(self, q, k, v, dense=False, out=None):
        """q, k, v [B,H,N,d] (original order) -> attention output [B,H,N,d] in ``out``
        (default: a buffer owned by the path, overwritten by the next call)."""
        if dense:
            fvattn_permute(q, self.qp, self.grid)
            fvattn_permute(k, self.kp, self.grid)
        else:
            self.route(q, k)
        self.prepare_v(v)
        self.attend(dense=dense)
        dst = self.out if out is None else out
        fvattn_permute(self.op, dst, self.grid, inverse=True)
        return dst

    def capture_graph(self, q, k, v, dense=False, out=None):
        """Captures one whole call on the given tensors into a CUDA graph (the
        library allocates nothing and never synchronizes the host inside a call,
        so every step is capturable). ``graph.replay()`` re-runs it on whatever q,
        k, v hold at that time. Returns (graph, output tensor)."""
        dst = self.out if out is None else out
        return _capture(self, q, k, v, dense, dst), dst


def _capture(path, q, k, v, dense, out):
    dev = path.qp.device
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):          # first launches (kernel attributes) outside the capture
        path(q, k, v, dense=dense, out=out)
    torch.cuda.current_stream(dev).wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        path(q, k, v, dense=dense, out=out)
    return graph


class HostPipeline:
    """Runs an FVAttnPath over a sequence of calls whose q, k, v live in pinned host
    memory and whose outputs go back to pinned host memory, with the copies of
    neighbouring calls overlapping the kernels of the current one.

    Two device input sets and two output buffers alternate. Uploads run on one
    copy stream, downloads on another. Events order them: call i's kernels wait
    for its upload; its download waits for its kernels; the upload of call i+2
    waits until call i's kernels have read the shared input set; call i+2's
    kernels wait until call i's download has read the shared output buffer.

    ``head_groups`` > 1 (B == 1) runs every call as that many head ranges, each on
    its own stream with its own sub-path (FVAttnPath.split_heads), with the same
    ordering per range. The heads are independent, so the results are the same;
    the first range's kernels start after a fraction of the first upload, and the
    last call's outputs start down as soon as each range is done.
    """

    def __init__(self, path: FVAttnPath, dense=False, head_groups=1):
        self.path = path
        self.dense = dense
        dev = path.qp.device
        self.device = dev
        shp = (path.B, path.H, path.N, path.d)
        self.inp = [tuple(torch.empty(shp, dtype=path.dtype, device=dev) for _ in range(3)) for _ in range(2)]
        self.outp = [torch.empty(shp, dtype=path.dtype, device=dev) for _ in range(2)]
        self.up = torch.cuda.Stream(device=dev)
        self.down = torch.cuda.Stream(device=dev)
        if head_groups > 1:
            self.parts = path.split_heads(head_groups)
            self.streams = [torch.cuda.Stream(device=dev) for _ in self.parts]
        else:
            self.parts = [(0, path.H, path)]
            self.streams = [None]             # the caller's current stream
        self._ev = lambda: torch.cuda.Event()
        g = len(self.parts)
        self.done_read = [[None] * g for _ in range(2)]   # kernels of the last call on slot s read range g
        self.done_down = [[None] * g for _ in range(2)]   # download of the last call on slot s read range g

    def run(self, host_qkv, host_out, start_event=None):
        """host_qkv: sequence of (q, k, v) pinned CPU tensors; host_out: sequence of
        pinned CPU tensors (may repeat). Enqueues every call; returns the event
        recorded on the current stream after the last download."""
        cur = torch.cuda.current_stream(self.device)
        comps = [st if st is not None else cur for st in self.streams]
        if start_event is not None:
            self.up.wait_event(start_event)
            self.down.wait_event(start_event)
        last = [None] * len(self.parts)
        for i, ((hq, hk, hv), ho) in enumerate(zip(host_qkv, host_out)):
            s = i & 1
            dq, dk, dv = self.inp[s]
            for g, (h0, h1, sub) in enumerate(self.parts):
                hs = slice(h0, h1)
                with torch.cuda.stream(self.up):
                    if self.done_read[s][g] is not None:
                        self.up.wait_event(self.done_read[s][g])
                    dq[:, hs].copy_(hq[:, hs], non_blocking=True)
                    dk[:, hs].copy_(hk[:, hs], non_blocking=True)
                    dv[:, hs].copy_(hv[:, hs], non_blocking=True)
                    ev_in = self._ev()
                    ev_in.record(self.up)
                comp = comps[g]
                comp.wait_event(ev_in)
                if self.done_down[s][g] is not None:
                    comp.wait_event(self.done_down[s][g])
                with torch.cuda.stream(comp):
                    sub(dq[:, hs], dk[:, hs], dv[:, hs], dense=self.dense, out=self.outp[s][:, hs])
                    ev_k = self._ev()
                    ev_k.record(comp)
                self.done_read[s][g] = ev_k
                with torch.cuda.stream(self.down):
                    self.down.wait_event(ev_k)
                    ho[:, hs].copy_(self.outp[s][:, hs], non_blocking=True)
                    ev_d = self._ev()
                    ev_d.record(self.down)
                self.done_down[s][g] = ev_d
                last[g] = ev_d
        for e in last:
            if e is not None:
                cur.wait_event(e)
        end = self._ev()
        end.record(cur)
        return end
