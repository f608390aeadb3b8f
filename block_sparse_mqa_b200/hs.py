"""Thin ctypes binding of libhs (include/hs.h), the sm_100a HySparse MQA
forward library.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory (tensors allocated here for outputs
and workspace) and the current CUDA stream.  There is no CPU fallback: when
``libhs.so`` is missing every call raises.

Function names match the C entry points.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhs.so")

HS_OK = 0
HS_ERR_INVALID_ARG = 1
HS_ERR_UNSUPPORTED = 2
HS_ERR_CUDA = 3
HS_ERR_INVALID_INDEX = 4
HS_ERR_TIMEOUT = 5
HS_ERR_WORKSPACE = 6

HS_F32 = 0
HS_BF16 = 1

HS_OP_BLOCK_SCORE = 0
HS_OP_SELECT_TOPK = 1
HS_OP_SPARSE_MQA = 2
HS_OP_SWA_MQA = 3
HS_OP_SPARSE_MQA_BWD = 4
HS_OP_SWA_MQA_BWD = 5
HS_OP_BLOCK_SCORE_ATTN = 6
HS_OP_SWA_LAYER = 7

HS_PATH_SIMT = 0
HS_PATH_TCGEN05 = 1
HS_PATH_MMA = 2

# every symbol include/hs.h declares
EXPORTS = (
    "hs_block_score", "hs_select_topk", "hs_sparse_mqa_fwd", "hs_swa_mqa_fwd",
    "hs_workspace_size", "hs_path", "hs_poll_status", "hs_set_force_simt",
    "hs_selftest_wait", "hs_status_string", "hs_last_error", "hs_version",
    "hs_block_score_static", "hs_sparse_mqa_bwd", "hs_swa_mqa_bwd",
    "hs_block_score_attn_fwd", "hs_swa_layer_fwd", "hs_last_path",
)


class HSError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("%s: %s" % (_status_name(status), msg))
        self.status = status


_lib = None
_i64 = ctypes.c_int64
_int = ctypes.c_int
_vp = ctypes.c_void_p
_flt = ctypes.c_float
_szt = ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """Load libhs.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libhs.so is not built (python -m block_sparse_mqa_b200.build); "
                           "there is no fallback implementation")
    L = ctypes.CDLL(LIB_PATH)
    L.hs_block_score.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _int, _int, _int, _int, _int,
                                 _int, _flt, _int, _vp, _vp, _int, _vp, _vp, _szt, _vp]
    L.hs_block_score_static.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _int, _int, _int, _int,
                                        _int, _int, _flt, _int, _vp, _vp, _int, _vp, _vp]
    L.hs_select_topk.argtypes = [_vp, _int, _vp, _int, _int, _int, _int, _int, _vp, _vp]
    L.hs_sparse_mqa_fwd.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _int, _int, _int,
                                    _int, _int, _int, _int, _flt, _vp, _int, _int, _vp, _vp, _vp,
                                    _vp]
    L.hs_swa_mqa_fwd.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _int, _int, _int,
                                 _int, _int, _int, _int, _flt, _int, _vp, _vp, _vp, _vp]
    L.hs_sparse_mqa_bwd.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _int, _int, _int,
                                    _int, _int, _int, _int, _flt, _vp, _int, _int, _vp, _vp, _vp,
                                    _vp, _vp, _vp, _vp, _vp, _vp, _szt, _vp]
    L.hs_swa_mqa_bwd.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _int, _int, _int,
                                 _int, _int, _int, _int, _flt, _int, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _vp, _vp, _vp, _szt, _vp]
    L.hs_block_score_attn_fwd.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _int, _int,
                                          _int, _int, _int, _int, _int, _flt, _int, _vp, _vp,
                                          _vp, _int, _vp, _vp, _szt, _vp]
    L.hs_swa_layer_fwd.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _i64, _vp, _i64,
                                   _vp, _int, _int, _int, _int, _int, _int, _int, _flt, _int,
                                   _vp, _vp, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    L.hs_workspace_size.argtypes = [_int] * 9
    L.hs_workspace_size.restype = _szt
    L.hs_path.argtypes = [_int] * 6
    L.hs_poll_status.argtypes = [_vp]
    L.hs_set_force_simt.argtypes = [_int]
    L.hs_set_force_simt.restype = None
    L.hs_selftest_wait.argtypes = [ctypes.c_longlong, _vp]
    L.hs_selftest_wait.restype = _int
    L.hs_status_string.argtypes = [_int]
    L.hs_status_string.restype = ctypes.c_char_p
    L.hs_last_error.argtypes = []
    L.hs_last_error.restype = ctypes.c_char_p
    L.hs_last_path.argtypes = []
    L.hs_last_path.restype = _int
    for fn in ("hs_block_score", "hs_select_topk", "hs_sparse_mqa_fwd", "hs_swa_mqa_fwd",
               "hs_poll_status", "hs_block_score_static", "hs_sparse_mqa_bwd",
               "hs_swa_mqa_bwd", "hs_block_score_attn_fwd", "hs_swa_layer_fwd"):
        getattr(L, fn).restype = _int
    _lib = L
    return L


def _status_name(st: int) -> str:
    try:
        return lib().hs_status_string(st).decode()
    except Exception:  # library not loadable while formatting an error
        return "status %d" % st


def _check(st: int):
    if st != HS_OK:
        raise HSError(st, lib().hs_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HS_BF16
    if t.dtype == torch.float32:
        return HS_F32
    raise TypeError("q/k/v must be bfloat16 or float32, got %s" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (libhs has no CPU path)")


def _qk_strides(q, k):
    if q.dim() != 3 or k.dim() != 2:
        raise ValueError("q must be [T, H, Dk] and k [T, Dk]")
    if q.stride(2) != 1 or k.stride(1) != 1:
        raise ValueError("innermost dimension of q and k must be contiguous")
    return q.stride(0), q.stride(1), k.stride(0)


def set_force_simt(on: bool):
    lib().hs_set_force_simt(1 if on else 0)


def selftest_wait(limit_ns: int, device=None):
    """Launch the bounded-wait self test (see include/hs.h)."""
    dev = torch.device("cuda" if device is None else device)
    _check(lib().hs_selftest_wait(int(limit_ns), _stream(dev)))


def path(op: int, dtype: torch.dtype, num_heads: int, dk: int, dv: int, block_size: int) -> int:
    code = HS_BF16 if dtype == torch.bfloat16 else HS_F32
    return lib().hs_path(op, code, num_heads, dk, dv, block_size)


def last_path() -> int:
    """Kernel family the calling thread's most recent successful call ran
    (HS_PATH_*), -1 before the first one: tells a call that left the
    tensor-core path because of its pointers or strides."""
    return int(lib().hs_last_path())


def poll_status(device=None):
    dev = torch.device("cuda" if device is None else device)
    _check(lib().hs_poll_status(_stream(dev)))


def workspace_size(op, total_tokens, num_docs, max_seqlen, num_heads, dk, dv, dtype, block_size):
    code = HS_BF16 if dtype == torch.bfloat16 else HS_F32
    return int(lib().hs_workspace_size(op, total_tokens, num_docs, max_seqlen, num_heads, dk, dv,
                                       code, block_size))


def nbmax(max_seqlen: int, block_size: int) -> int:
    return (max_seqlen + block_size - 1) // block_size


def _check_block_outputs(bs, blse, T, H, nb):
    """block_score [T, nb_stride] and block_lse [T, H, nb_stride] share one
    column stride (nb_stride >= NBmax) in the C calls."""
    if bs.dtype != torch.float32 or bs.dim() != 2 or bs.shape[0] != T or bs.stride(1) != 1 \
            or bs.stride(0) < nb or bs.shape[1] < nb:
        raise ValueError("block_score must be float32 [T, >= NBmax] with contiguous rows")
    if blse is not None:
        ns = bs.stride(0)
        if blse.dtype != torch.float32 or tuple(blse.shape) != (T, H, ns) or \
                not blse.is_contiguous():
            raise ValueError("block_lse must be contiguous float32 [T, H, nb_stride] with the "
                             "block_score row stride")


def hs_block_score(q, k, cu_seqlens, max_seqlen: int, block_size: int,
                   softmax_scale: float = 0.0, want_block_lse: bool = False,
                   out_lse=None, out_block_score=None, out_block_lse=None, workspace=None):
    """Step 1.  Returns (lse [T,H] f32, block_score [T,NBmax] f32,
    block_lse [T,H,NBmax] f32 or None)."""
    _need_cuda(q, k, cu_seqlens)
    qrs, qhs, krs = _qk_strides(q, k)
    T, H, Dk = q.shape
    nb = nbmax(max_seqlen, block_size)
    dev = q.device
    f32 = torch.float32
    lse = out_lse if out_lse is not None else torch.empty((T, H), device=dev, dtype=f32)
    bs = out_block_score if out_block_score is not None else torch.empty((T, nb), device=dev, dtype=f32)
    blse = out_block_lse
    if want_block_lse and blse is None:
        blse = torch.empty((T, H, nb), device=dev, dtype=f32)
    _check_block_outputs(bs, blse, T, H, nb)
    nd = cu_seqlens.numel() - 1
    need = workspace_size(HS_OP_BLOCK_SCORE, T, nd, max_seqlen, H, Dk, 0, q.dtype, block_size)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    _check(lib().hs_block_score(
        _ptr(q), qrs, qhs, _ptr(k), krs, _ptr(cu_seqlens), nd, T, int(max_seqlen), H, Dk,
        _dtype_code(q), float(softmax_scale), int(block_size), _ptr(lse), _ptr(bs), bs.stride(0),
        _ptr(blse), _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream(dev)))
    return lse, bs, blse


def hs_block_score_static(q, k, cu_seqlens, max_seqlen: int, block_size: int,
                          softmax_scale: float = 0.0, want_block_lse: bool = False):
    """Step 1 without a workspace: for callers that cannot allocate device
    memory, the library's fixed 16 MiB scratch array is used instead (see
    include/hs.h for the size limit and the one-call-at-a-time rule).  The
    output tensors here are allocated by torch for convenience; a caller that
    cannot allocate passes its own output pointers to the C entry point."""
    _need_cuda(q, k, cu_seqlens)
    qrs, qhs, krs = _qk_strides(q, k)
    T, H, Dk = q.shape
    nb = nbmax(max_seqlen, block_size)
    dev = q.device
    lse = torch.empty((T, H), device=dev, dtype=torch.float32)
    bs = torch.empty((T, nb), device=dev, dtype=torch.float32)
    blse = torch.empty((T, H, nb), device=dev, dtype=torch.float32) if want_block_lse else None
    _check(lib().hs_block_score_static(
        _ptr(q), qrs, qhs, _ptr(k), krs, _ptr(cu_seqlens), cu_seqlens.numel() - 1, T,
        int(max_seqlen), H, Dk, _dtype_code(q), float(softmax_scale), int(block_size), _ptr(lse),
        _ptr(bs), bs.stride(0), _ptr(blse), _stream(dev)))
    return lse, bs, blse


def hs_select_topk(block_score, cu_seqlens, max_seqlen: int, block_size: int, topk: int,
                   out_idx=None):
    """Step 2.  Returns idx [T, topk] int32 (ascending, -1 padded)."""
    _need_cuda(block_score, cu_seqlens)
    if block_score.dtype != torch.float32 or block_score.stride(1) != 1:
        raise ValueError("block_score must be float32 with contiguous rows")
    T = block_score.shape[0]
    idx = out_idx if out_idx is not None else torch.empty((T, topk), device=block_score.device,
                                                          dtype=torch.int32)
    _check(lib().hs_select_topk(
        _ptr(block_score), block_score.stride(0), _ptr(cu_seqlens), cu_seqlens.numel() - 1, T,
        int(max_seqlen), int(block_size), int(topk), _ptr(idx), _stream(block_score.device)))
    return idx


def _attn_out(q, v, out, lse):
    T, H, _ = q.shape
    Dv = v.shape[1]
    o = out if out is not None else torch.empty((T, H, Dv), device=q.device, dtype=q.dtype)
    l = lse if lse is not None else torch.empty((T, H), device=q.device, dtype=torch.float32)
    if not o.is_contiguous() or not l.is_contiguous():
        raise ValueError("out and lse must be contiguous")
    return o, l


def hs_sparse_mqa_fwd(q, k, v, idx, cu_seqlens, max_seqlen: int, block_size: int,
                      sink=None, softmax_scale: float = 0.0, out=None, lse=None):
    """Step 3.  Returns (out [T,H,Dv] in q's dtype, lse [T,H] f32)."""
    _need_cuda(q, k, v, idx, cu_seqlens, sink)
    qrs, qhs, krs = _qk_strides(q, k)
    if v.dim() != 2 or v.stride(1) != 1:
        raise ValueError("v must be [T, Dv] with contiguous rows")
    if idx.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx must be contiguous int32 [T, topk]")
    T, H, Dk = q.shape
    o, l = _attn_out(q, v, out, lse)
    _check(lib().hs_sparse_mqa_fwd(
        _ptr(q), qrs, qhs, _ptr(k), krs, _ptr(v), v.stride(0), _ptr(cu_seqlens),
        cu_seqlens.numel() - 1, T, int(max_seqlen), H, Dk, v.shape[1], _dtype_code(q),
        float(softmax_scale), _ptr(idx), idx.shape[1], int(block_size), _ptr(sink), _ptr(o),
        _ptr(l), _stream(q.device)))
    return o, l


def hs_swa_mqa_fwd(q, k, v, cu_seqlens, max_seqlen: int, window: int, sink=None,
                   softmax_scale: float = 0.0, out=None, lse=None):
    """Step 4.  Returns (out [T,H,Dv] in q's dtype, lse [T,H] f32)."""
    _need_cuda(q, k, v, cu_seqlens, sink)
    qrs, qhs, krs = _qk_strides(q, k)
    if v.dim() != 2 or v.stride(1) != 1:
        raise ValueError("v must be [T, Dv] with contiguous rows")
    T, H, Dk = q.shape
    o, l = _attn_out(q, v, out, lse)
    _check(lib().hs_swa_mqa_fwd(
        _ptr(q), qrs, qhs, _ptr(k), krs, _ptr(v), v.stride(0), _ptr(cu_seqlens),
        cu_seqlens.numel() - 1, T, int(max_seqlen), H, Dk, v.shape[1], _dtype_code(q),
        float(softmax_scale), int(window), _ptr(sink), _ptr(o), _ptr(l), _stream(q.device)))
    return o, l


def hs_block_score_attn_fwd(q, k, v, cu_seqlens, max_seqlen: int, block_size: int,
                            softmax_scale: float = 0.0, want_block_lse: bool = False, out=None,
                            lse=None, out_block_score=None, out_block_lse=None, workspace=None):
    """The full layer's forward with step 1 fused in: dense causal attention
    (no sink) plus step 1's outputs.  Returns (out [T,H,Dv] in q's dtype,
    lse [T,H] f32, block_score [T,NBmax] f32, block_lse [T,H,NBmax] f32 or
    None)."""
    _need_cuda(q, k, v, cu_seqlens)
    qrs, qhs, krs = _qk_strides(q, k)
    if v.dim() != 2 or v.stride(1) != 1:
        raise ValueError("v must be [T, Dv] with contiguous rows")
    T, H, Dk = q.shape
    Dv = v.shape[1]
    o, l = _attn_out(q, v, out, lse)
    nb = nbmax(max_seqlen, block_size)
    dev = q.device
    bs = out_block_score if out_block_score is not None else torch.empty(
        (T, nb), device=dev, dtype=torch.float32)
    blse = out_block_lse
    if want_block_lse and blse is None:
        blse = torch.empty((T, H, nb), device=dev, dtype=torch.float32)
    _check_block_outputs(bs, blse, T, H, nb)
    nd = cu_seqlens.numel() - 1
    need = workspace_size(HS_OP_BLOCK_SCORE_ATTN, T, nd, max_seqlen, H, Dk, Dv, q.dtype,
                          block_size)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    _check(lib().hs_block_score_attn_fwd(
        _ptr(q), qrs, qhs, _ptr(k), krs, _ptr(v), v.stride(0), _ptr(cu_seqlens), nd, T,
        int(max_seqlen), H, Dk, Dv, _dtype_code(q), float(softmax_scale), int(block_size),
        _ptr(o), _ptr(l), _ptr(bs), bs.stride(0), _ptr(blse), _ptr(workspace),
        0 if workspace is None else workspace.numel(), _stream(dev)))
    return o, l, bs, blse


def hs_swa_layer_fwd(q, k, v, k_shared, v_shared, idx, cu_seqlens, max_seqlen: int, window: int,
                     block_size: int, sink_swa=None, sink_sparse=None, gate_swa=None,
                     gate_sparse=None, softmax_scale: float = 0.0, out=None, lse_swa=None,
                     lse_sparse=None):
    """The SWA layer: window attention over its own k, v plus the sparse
    branch over the full layer's k_shared, v_shared and block lists idx,
    combined as gate_swa * window + gate_sparse * sparse (missing gates = 1).
    Returns (out [T,H,Dv] in q's dtype, lse_swa [T,H], lse_sparse [T,H])."""
    _need_cuda(q, k, v, k_shared, v_shared, idx, cu_seqlens, sink_swa, sink_sparse, gate_swa,
               gate_sparse)
    qrs, qhs, krs = _qk_strides(q, k)
    _, _, ksrs = _qk_strides(q, k_shared)
    for name, t in (("v", v), ("v_shared", v_shared)):
        if t.dim() != 2 or t.stride(1) != 1:
            raise ValueError(name + " must be [T, Dv] with contiguous rows")
    if idx.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx must be contiguous int32 [T, topk]")
    T, H, Dk = q.shape
    for name, g in (("gate_swa", gate_swa), ("gate_sparse", gate_sparse)):
        if g is not None and (g.dtype != torch.float32 or tuple(g.shape) != (T, H) or
                              not g.is_contiguous()):
            raise ValueError(name + " must be contiguous float32 [T, H]")
    o, lw = _attn_out(q, v, out, lse_swa)
    ls = lse_sparse if lse_sparse is not None else torch.empty_like(lw)
    _check(lib().hs_swa_layer_fwd(
        _ptr(q), qrs, qhs, _ptr(k), krs, _ptr(v), v.stride(0), _ptr(k_shared), ksrs,
        _ptr(v_shared), v_shared.stride(0), _ptr(cu_seqlens), cu_seqlens.numel() - 1, T,
        int(max_seqlen), H, Dk, v.shape[1], _dtype_code(q), float(softmax_scale), int(window),
        _ptr(sink_swa), _ptr(idx), idx.shape[1], int(block_size), _ptr(sink_sparse),
        _ptr(gate_swa), _ptr(gate_sparse), _ptr(o), _ptr(lw), _ptr(ls), _stream(q.device)))
    return o, lw, ls


def _bwd_prep(q, k, v, out, lse, dout, cu_seqlens, sink, op, max_seqlen, grads, workspace):
    _need_cuda(q, k, v, out, lse, dout, cu_seqlens, sink)
    qrs, qhs, krs = _qk_strides(q, k)
    if v.dim() != 2 or v.stride(1) != 1:
        raise ValueError("v must be [T, Dv] with contiguous rows")
    for name, t in (("out", out), ("lse", lse), ("dout", dout)):
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous" % name)
    if lse.dtype != torch.float32 or out.dtype != q.dtype or dout.dtype != q.dtype:
        raise ValueError("lse must be float32; out and dout in q's dtype")
    T, H, Dk = q.shape
    Dv = v.shape[1]
    dev = q.device
    f32 = torch.float32
    if grads is None:
        grads = (torch.empty((T, H, Dk), device=dev, dtype=f32),
                 torch.empty((T, Dk), device=dev, dtype=f32),
                 torch.empty((T, Dv), device=dev, dtype=f32),
                 torch.empty((H,), device=dev, dtype=f32) if sink is not None else None)
    for g in grads:
        if g is not None and (g.dtype != f32 or not g.is_contiguous()):
            raise ValueError("gradient outputs must be contiguous float32")
    need = workspace_size(op, T, cu_seqlens.numel() - 1, max_seqlen, H, Dk, Dv, q.dtype, 64)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    return qrs, qhs, krs, grads, workspace


def hs_sparse_mqa_bwd(q, k, v, idx, cu_seqlens, max_seqlen: int, block_size: int, out, lse,
                      dout, sink=None, softmax_scale: float = 0.0, grads=None, workspace=None):
    """Backward of step 3.  Returns (dq [T,H,Dk], dk [T,Dk], dv [T,Dv],
    dsink [H] or None), all float32."""
    if idx.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx must be contiguous int32 [T, topk]")
    qrs, qhs, krs, g, ws = _bwd_prep(q, k, v, out, lse, dout, cu_seqlens, sink,
                                     HS_OP_SPARSE_MQA_BWD, max_seqlen, grads, workspace)
    T, H, Dk = q.shape
    _check(lib().hs_sparse_mqa_bwd(
        _ptr(q), qrs, qhs, _ptr(k), krs, _ptr(v), v.stride(0), _ptr(cu_seqlens),
        cu_seqlens.numel() - 1, T, int(max_seqlen), H, Dk, v.shape[1], _dtype_code(q),
        float(softmax_scale), _ptr(idx), idx.shape[1], int(block_size), _ptr(sink), _ptr(out),
        _ptr(lse), _ptr(dout), _ptr(g[0]), _ptr(g[1]), _ptr(g[2]), _ptr(g[3]), _ptr(ws),
        0 if ws is None else ws.numel(), _stream(q.device)))
    return g


def hs_swa_mqa_bwd(q, k, v, cu_seqlens, max_seqlen: int, window: int, out, lse, dout,
                   sink=None, softmax_scale: float = 0.0, grads=None, workspace=None):
    """Backward of step 4.  Returns (dq, dk, dv, dsink or None), float32."""
    qrs, qhs, krs, g, ws = _bwd_prep(q, k, v, out, lse, dout, cu_seqlens, sink,
                                     HS_OP_SWA_MQA_BWD, max_seqlen, grads, workspace)
    T, H, Dk = q.shape
    _check(lib().hs_swa_mqa_bwd(
        _ptr(q), qrs, qhs, _ptr(k), krs, _ptr(v), v.stride(0), _ptr(cu_seqlens),
        cu_seqlens.numel() - 1, T, int(max_seqlen), H, Dk, v.shape[1], _dtype_code(q),
        float(softmax_scale), int(window), _ptr(sink), _ptr(out), _ptr(lse), _ptr(dout),
        _ptr(g[0]), _ptr(g[1]), _ptr(g[2]), _ptr(g[3]), _ptr(ws),
        0 if ws is None else ws.numel(), _stream(q.device)))
    return g


def hs_forward(q, k, v, cu_seqlens, max_seqlen: int, block_size: int, topk: int, window: int,
               sink=None, softmax_scale: float = 0.0, with_swa: bool = True):
    """The whole forward path: score -> select -> sparse attention (and the
    sliding-window attention over the same q, k, v).  Returns a dict."""
    lse1, bs, _ = hs_block_score(q, k, cu_seqlens, max_seqlen, block_size, softmax_scale)
    idx = hs_select_topk(bs, cu_seqlens, max_seqlen, block_size, topk)
    out, lse = hs_sparse_mqa_fwd(q, k, v, idx, cu_seqlens, max_seqlen, block_size, sink,
                                 softmax_scale)
    res = {"score_lse": lse1, "block_score": bs, "idx": idx, "sparse_out": out,
           "sparse_lse": lse}
    if with_swa:
        res["swa_out"], res["swa_lse"] = hs_swa_mqa_fwd(q, k, v, cu_seqlens, max_seqlen, window,
                                                        sink, softmax_scale)
    return res
