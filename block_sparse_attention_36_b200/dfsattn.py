"""Python binding of libdfsattn (argument marshalling only).

Every function forwards to the C entry point of the same name declared in
include/dfsattn.h; each stage of the path runs in the library's CUDA
kernels. torch tensors supply device memory and the current CUDA stream.
There is no fallback: if the library is missing or fails to load, importing
this module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdfsattn.so")

DFS_OK = 0
DFS_ERR_INVALID_ARG = -1
DFS_ERR_UNSUPPORTED = -2
DFS_ERR_MISALIGNED = -3
DFS_ERR_CUDA = -4
DFS_ERR_TIMEOUT = -5
DFS_ERR_WORKSPACE = -6

DFS_ORDER_RASTER = 0
DFS_ORDER_HILBERT3D = 1
DFS_SEL_TOPK = 0
DFS_SEL_THRESHOLD = 1
DFS_SEL_LVSA = 2
DFS_SEL_GLOBAL = 3
DFS_SEL_RADIAL = 4
DFS_WS_BLOCK_SCORE = 0
DFS_WS_ATTN_BWD = 1

DFS_FLAG_WAIT_TIMEOUT = 1
DFS_FLAG_BAD_KV_INDEX = 2
DFS_FLAG_KCAP_OVERFLOW = 4

DFS_ORDER_TILE2D = 2
DFS_ORDER_TILE3D = 3
DFS_ORDER_HILBERT2D = 4
ORDERS = {"raster": DFS_ORDER_RASTER, "hilbert3d": DFS_ORDER_HILBERT3D, "tile2d": DFS_ORDER_TILE2D,
          "tile3d": DFS_ORDER_TILE3D, "hilbert2d": DFS_ORDER_HILBERT2D}
MODES = {"topk": DFS_SEL_TOPK, "threshold": DFS_SEL_THRESHOLD, "lvsa": DFS_SEL_LVSA, "global": DFS_SEL_GLOBAL,
         "radial": DFS_SEL_RADIAL}

# C entry points declared in include/dfsattn.h.
EXPORTS = (
    "dfs_hilbert_perm", "dfs_block_score", "dfs_select_mask", "dfs_sparse_attn_fwd", "dfs_unperm",
    "dfs_workspace_bytes", "dfs_get_error_flags", "dfs_status_string", "dfs_version", "dfs_block_score_noalloc",
    "dfs_hilbert_perm_pooled", "dfs_block_score_pooled", "dfs_sparse_attn_lvsa_fwd", "dfs_sparse_attn_bwd",
    "dfs_sparse_attn_fwd_ex", "dfs_attn_order",
)


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "nh", "D", "T", "H", "W", "blk", "sb")]


class _AttnOpts(ctypes.Structure):
    _fields_ = [("perm", ctypes.c_void_p), ("order", ctypes.c_void_p), ("no_tail_split", ctypes.c_int),
                ("test_stall_cycles", ctypes.c_uint)]


class _SelectParams(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("k", ctypes.c_int), ("cap", ctypes.c_int), ("tau", ctypes.c_float),
                ("lvsa_T_per", ctypes.c_int), ("lvsa_C", ctypes.c_int), ("lvsa_step", ctypes.c_int),
                ("radial_w0", ctypes.c_int), ("radial_lambda", ctypes.c_float)]


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libdfsattn.so is not built ({_LIB_PATH}); run "
                          "python -m block_sparse_attention_36_b200.build")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sp = ctypes.POINTER(_Shape)
    lib.dfs_hilbert_perm.argtypes = [sp, I, P, P, I, P, P, P, P, P, P, P]
    lib.dfs_block_score.argtypes = [sp, P, P, F, P, P, S, P]
    lib.dfs_select_mask.argtypes = [sp, P, ctypes.POINTER(_SelectParams), P, P, I, P]
    lib.dfs_block_score_noalloc.argtypes = [sp, P, P, F, P, P]
    lib.dfs_hilbert_perm_pooled.argtypes = [sp, I, P, P, I, P, P, P, P, P, P, P, S, P]
    lib.dfs_block_score_pooled.argtypes = [sp, F, P, P, S, P]
    lib.dfs_sparse_attn_lvsa_fwd.argtypes = [sp, P, P, P, P, P, I, F, ctypes.POINTER(_SelectParams), P, P, P]
    lib.dfs_sparse_attn_bwd.argtypes = [sp, P, P, P, P, P, P, P, P, I, F, P, P, P, P, S, P]
    lib.dfs_sparse_attn_fwd_ex.argtypes = [sp, P, P, P, P, P, I, F, ctypes.POINTER(_AttnOpts), P, P, P]
    lib.dfs_attn_order.argtypes = [sp, P, I, P, P]
    lib.dfs_sparse_attn_fwd.argtypes = [sp, P, P, P, P, P, I, F, P, P, P]
    lib.dfs_unperm.argtypes = [sp, P, P, P, P]
    lib.dfs_workspace_bytes.argtypes = [sp, I]
    lib.dfs_workspace_bytes.restype = S
    lib.dfs_get_error_flags.argtypes = [ctypes.POINTER(ctypes.c_uint32), I]
    lib.dfs_status_string.argtypes = [I]
    lib.dfs_status_string.restype = ctypes.c_char_p
    lib.dfs_version.argtypes = []
    for name in ("dfs_hilbert_perm", "dfs_block_score", "dfs_select_mask", "dfs_sparse_attn_fwd",
                 "dfs_unperm", "dfs_get_error_flags", "dfs_version", "dfs_block_score_noalloc",
                 "dfs_hilbert_perm_pooled", "dfs_block_score_pooled", "dfs_sparse_attn_lvsa_fwd",
                 "dfs_sparse_attn_bwd", "dfs_sparse_attn_fwd_ex", "dfs_attn_order"):
        getattr(lib, name).restype = I
    return lib


LIB = _load()


class DfsError(RuntimeError):
    def __init__(self, call, status, detail=None):
        msg = f"{call}: {LIB.dfs_status_string(status).decode()} ({status})"
        super().__init__(msg if detail is None else f"{msg}: {detail}")
        self.status = status


def _check(call, status):
    if status != DFS_OK:
        raise DfsError(call, status)


def _need(call, name, t, numel, dtype, optional=False):
    """Host check of one tensor argument before its pointer goes to C: a CUDA
    tensor of the expected dtype, contiguous, holding at least ``numel``
    elements (the size the shape implies). The C side cannot see sizes, so a
    wrong tensor would otherwise become an out-of-bounds device access."""
    if t is None:
        if optional:
            return
        raise DfsError(call, DFS_ERR_INVALID_ARG, f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise DfsError(call, DFS_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise DfsError(call, DFS_ERR_INVALID_ARG, f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise DfsError(call, DFS_ERR_INVALID_ARG, f"{name} must be contiguous")
    if t.numel() < numel:
        raise DfsError(call, DFS_ERR_INVALID_ARG, f"{name} holds {t.numel()} elements, the shape needs {numel}")


def _need_ws(call, ws):
    """A workspace may have any dtype (its size in bytes is checked by the C
    side), but it must be contiguous device memory."""
    if ws is not None and (not isinstance(ws, torch.Tensor) or not ws.is_cuda or not ws.is_contiguous()):
        raise DfsError(call, DFS_ERR_INVALID_ARG, "ws must be a contiguous CUDA tensor")


_BF16, _F32, _I32 = torch.bfloat16, torch.float32, torch.int32


def _tok(shape):      # elements of one [B, N, nh, D] / [B, nh, N, D] tensor
    return shape.B * shape.nh * shape.N * shape.D


def _rows(shape):     # query rows (b, h, I)
    return shape.B * shape.nh * shape.nb


@dataclass(frozen=True)
class Shape:
    B: int
    nh: int
    D: int
    T: int
    H: int
    W: int
    blk: int
    sb: int

    @property
    def N(self):
        return self.T * self.H * self.W

    @property
    def nb(self):
        return -(-self.N // self.blk)

    @property
    def nsb(self):
        return -(-self.N // self.sb)

    def c(self):
        return _Shape(self.B, self.nh, self.D, self.T, self.H, self.W, self.blk, self.sb)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def dfs_hilbert_perm(shape: Shape, order, perm, inv, build_index, q, k, v, qp, kp, vp, stream=None):
    order = ORDERS.get(order, order)
    c = "dfs_hilbert_perm"
    _need(c, "perm", perm, shape.N, _I32)
    _need(c, "inv", inv, shape.N, _I32, optional=not build_index)
    for n, t in (("q", q), ("k", k), ("v", v), ("qp", qp), ("kp", kp), ("vp", vp)):
        _need(c, n, t, _tok(shape), _BF16, optional=True)
    sh = shape.c()
    _check("dfs_hilbert_perm", LIB.dfs_hilbert_perm(
        ctypes.byref(sh), int(order), _ptr(perm), _ptr(inv), int(bool(build_index)),
        _ptr(q), _ptr(k), _ptr(v), _ptr(qp), _ptr(kp), _ptr(vp), _stream(stream)))


def dfs_hilbert_perm_pooled(shape: Shape, order, perm, inv, build_index, q, k, v, qp, kp, vp, ws, stream=None):
    order = ORDERS.get(order, order)
    c = "dfs_hilbert_perm_pooled"
    _need(c, "perm", perm, shape.N, _I32)
    _need(c, "inv", inv, shape.N, _I32, optional=not build_index)
    for n, t in (("q", q), ("k", k), ("qp", qp), ("kp", kp)):
        _need(c, n, t, _tok(shape), _BF16)
    for n, t in (("v", v), ("vp", vp)):
        _need(c, n, t, _tok(shape), _BF16, optional=True)
    _need_ws(c, ws)
    sh = shape.c()
    _check("dfs_hilbert_perm_pooled", LIB.dfs_hilbert_perm_pooled(
        ctypes.byref(sh), int(order), _ptr(perm), _ptr(inv), int(bool(build_index)),
        _ptr(q), _ptr(k), _ptr(v), _ptr(qp), _ptr(kp), _ptr(vp), _ptr(ws), _nbytes(ws),
        _stream(stream)))


def dfs_block_score_pooled(shape: Shape, scale, scores, ws, stream=None):
    _need("dfs_block_score_pooled", "scores", scores, _rows(shape) * shape.nb, _F32)
    _need_ws("dfs_block_score_pooled", ws)
    sh = shape.c()
    _check("dfs_block_score_pooled", LIB.dfs_block_score_pooled(
        ctypes.byref(sh), float(scale), _ptr(scores), _ptr(ws), _nbytes(ws),
        _stream(stream)))


def dfs_workspace_bytes(shape: Shape, which=DFS_WS_BLOCK_SCORE) -> int:
    sh = shape.c()
    return int(LIB.dfs_workspace_bytes(ctypes.byref(sh), int(which)))


def dfs_block_score(shape: Shape, qp, kp, scale, scores, ws, stream=None):
    for n, t in (("qp", qp), ("kp", kp)):
        _need("dfs_block_score", n, t, _tok(shape), _BF16)
    _need("dfs_block_score", "scores", scores, _rows(shape) * shape.nb, _F32)
    _need_ws("dfs_block_score", ws)
    sh = shape.c()
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("dfs_block_score", LIB.dfs_block_score(
        ctypes.byref(sh), _ptr(qp), _ptr(kp), float(scale), _ptr(scores), _ptr(ws), nbytes, _stream(stream)))


def dfs_block_score_noalloc(shape: Shape, qp, kp, scale, scores, stream=None):
    """dfs_block_score with the library's built-in scratch buffer instead of a
    workspace, for callers that cannot allocate device memory (see the C
    header for the size limit, first-call set-up and the sharing rule)."""
    for n, t in (("qp", qp), ("kp", kp)):
        _need("dfs_block_score_noalloc", n, t, _tok(shape), _BF16)
    _need("dfs_block_score_noalloc", "scores", scores, _rows(shape) * shape.nb, _F32)
    sh = shape.c()
    _check("dfs_block_score_noalloc", LIB.dfs_block_score_noalloc(
        ctypes.byref(sh), _ptr(qp), _ptr(kp), float(scale), _ptr(scores), _stream(stream)))


NOALLOC_SCRATCH_BYTES = 32 << 20


def select_params(mode, k=0, cap=0, tau=0.0, lvsa_T_per=8, lvsa_C=21, lvsa_step=0, radial_w0=0,
                  radial_lambda=0.0):
    return _SelectParams(MODES.get(mode, mode), int(k), int(cap), float(tau), int(lvsa_T_per), int(lvsa_C),
                         int(lvsa_step), int(radial_w0), float(radial_lambda))


def dfs_select_mask(shape: Shape, scores, params, kv_idx, kv_cnt, kcap, stream=None):
    c = "dfs_select_mask"
    _need(c, "scores", scores, _rows(shape) * shape.nb, _F32,
          optional=params.mode in (DFS_SEL_LVSA, DFS_SEL_RADIAL))
    _need(c, "kv_idx", kv_idx, _rows(shape) * max(1, int(kcap)), _I32)
    _need(c, "kv_cnt", kv_cnt, _rows(shape), _I32)
    sh = shape.c()
    _check("dfs_select_mask", LIB.dfs_select_mask(
        ctypes.byref(sh), _ptr(scores), ctypes.byref(params), _ptr(kv_idx), _ptr(kv_cnt), int(kcap),
        _stream(stream)))


def _need_attn(c, shape, qp, kp, vp, kv_idx, kv_cnt, kcap, o, lse):
    for n, t in (("qp", qp), ("kp", kp), ("vp", vp), ("o", o)):
        _need(c, n, t, _tok(shape), _BF16)
    _need(c, "kv_idx", kv_idx, _rows(shape) * max(1, int(kcap)), _I32)
    _need(c, "kv_cnt", kv_cnt, _rows(shape), _I32)
    _need(c, "lse", lse, shape.B * shape.nh * shape.N, _F32, optional=True)


def dfs_sparse_attn_fwd(shape: Shape, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse=None, stream=None):
    _need_attn("dfs_sparse_attn_fwd", shape, qp, kp, vp, kv_idx, kv_cnt, kcap, op, lse)
    sh = shape.c()
    _check("dfs_sparse_attn_fwd", LIB.dfs_sparse_attn_fwd(
        ctypes.byref(sh), _ptr(qp), _ptr(kp), _ptr(vp), _ptr(kv_idx), _ptr(kv_cnt), int(kcap), float(scale),
        _ptr(op), _ptr(lse), _stream(stream)))


def dfs_sparse_attn_fwd_ex(shape: Shape, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, o, lse=None, perm=None,
                           order=None, stream=None, tail_split=True, test_stall_cycles=0):
    c = "dfs_sparse_attn_fwd_ex"
    _need_attn(c, shape, qp, kp, vp, kv_idx, kv_cnt, kcap, o, lse)
    _need(c, "perm", perm, shape.N, _I32, optional=True)
    _need(c, "order", order, _rows(shape), _I32, optional=True)
    sh = shape.c()
    opts = _AttnOpts(None if perm is None else perm.data_ptr(), None if order is None else order.data_ptr(),
                     0 if tail_split else 1, int(test_stall_cycles))
    _check("dfs_sparse_attn_fwd_ex", LIB.dfs_sparse_attn_fwd_ex(
        ctypes.byref(sh), _ptr(qp), _ptr(kp), _ptr(vp), _ptr(kv_idx), _ptr(kv_cnt), int(kcap), float(scale),
        ctypes.byref(opts), _ptr(o), _ptr(lse), _stream(stream)))


def dfs_attn_order(shape: Shape, kv_cnt, kcap, order, stream=None):
    _need("dfs_attn_order", "kv_cnt", kv_cnt, _rows(shape), _I32)
    _need("dfs_attn_order", "order", order, _rows(shape), _I32)
    sh = shape.c()
    _check("dfs_attn_order", LIB.dfs_attn_order(ctypes.byref(sh), _ptr(kv_cnt), int(kcap), _ptr(order),
                                                _stream(stream)))


def dfs_sparse_attn_bwd(shape: Shape, qp, kp, vp, op, dop, lse, kv_idx, kv_cnt, kcap, scale, dqp, dkp, dvp, ws,
                        stream=None):
    c = "dfs_sparse_attn_bwd"
    for n, t in (("qp", qp), ("kp", kp), ("vp", vp), ("op", op), ("dop", dop), ("dqp", dqp), ("dkp", dkp),
                 ("dvp", dvp)):
        _need(c, n, t, _tok(shape), _BF16)
    _need(c, "lse", lse, shape.B * shape.nh * shape.N, _F32)
    _need(c, "kv_idx", kv_idx, _rows(shape) * max(1, int(kcap)), _I32)
    _need(c, "kv_cnt", kv_cnt, _rows(shape), _I32)
    _need_ws(c, ws)
    sh = shape.c()
    _check("dfs_sparse_attn_bwd", LIB.dfs_sparse_attn_bwd(
        ctypes.byref(sh), _ptr(qp), _ptr(kp), _ptr(vp), _ptr(op), _ptr(dop), _ptr(lse), _ptr(kv_idx), _ptr(kv_cnt),
        int(kcap), float(scale), _ptr(dqp), _ptr(dkp), _ptr(dvp), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def dfs_sparse_attn_lvsa_fwd(shape: Shape, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, params, op, lse=None,
                             stream=None):
    _need_attn("dfs_sparse_attn_lvsa_fwd", shape, qp, kp, vp, kv_idx, kv_cnt, kcap, op, lse)
    sh = shape.c()
    _check("dfs_sparse_attn_lvsa_fwd", LIB.dfs_sparse_attn_lvsa_fwd(
        ctypes.byref(sh), _ptr(qp), _ptr(kp), _ptr(vp), _ptr(kv_idx), _ptr(kv_cnt), int(kcap), float(scale),
        ctypes.byref(params), _ptr(op), _ptr(lse), _stream(stream)))


def dfs_unperm(shape: Shape, perm, op, o, stream=None):
    _need("dfs_unperm", "perm", perm, shape.N, _I32)
    _need("dfs_unperm", "op", op, _tok(shape), _BF16)
    _need("dfs_unperm", "o", o, _tok(shape), _BF16)
    sh = shape.c()
    _check("dfs_unperm", LIB.dfs_unperm(ctypes.byref(sh), _ptr(perm), _ptr(op), _ptr(o), _stream(stream)))


def dfs_get_error_flags(clear=True) -> int:
    v = ctypes.c_uint32(0)
    _check("dfs_get_error_flags", LIB.dfs_get_error_flags(ctypes.byref(v), int(bool(clear))))
    return int(v.value)


def dfs_version() -> int:
    return int(LIB.dfs_version())
