"""C-ABI checks that need no GPU: the library loads, exports every symbol
include/hs.h declares, and rejects bad arguments on the host before any CUDA
call (validation comes first, so these calls never touch a device)."""

import ctypes
import os
import re

import pytest

from block_sparse_mqa_b200 import hs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "hs.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hs_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = hs.lib()
    names = _declared()
    assert "hs_block_score" in names and "hs_swa_mqa_fwd" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(hs.EXPORTS)


def test_helpers():
    L = hs.lib()
    assert L.hs_version() >= 100
    assert L.hs_status_string(hs.HS_ERR_TIMEOUT) == b"HS_ERR_TIMEOUT"
    assert hs.path(hs.HS_OP_SELECT_TOPK, __import__("torch").float32, 4, 64, 48, 16) == hs.HS_PATH_SIMT
    assert L.hs_path(0, 7, 64, 576, 512, 64) == -1


_I64 = ctypes.c_int64
NULL = None


def _score(**kw):
    a = dict(q=1, qrs=64 * 576, qhs=576, k=1, krs=576, cu=1, nd=1, T=128, maxlen=128, H=64,
             dk=576, dt=hs.HS_BF16, scale=0.0, B=64, lse=1, bs=1, nbs=2, blse=NULL, ws=NULL,
             wsb=0)
    a.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return hs.lib().hs_block_score(v(a["q"]), a["qrs"], a["qhs"], v(a["k"]), a["krs"], v(a["cu"]),
                                   a["nd"], a["T"], a["maxlen"], a["H"], a["dk"], a["dt"],
                                   a["scale"], a["B"], v(a["lse"]), v(a["bs"]), a["nbs"],
                                   v(a["blse"]), v(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), hs.HS_ERR_INVALID_ARG),
    (dict(cu=None), hs.HS_ERR_INVALID_ARG),
    (dict(T=-1), hs.HS_ERR_INVALID_ARG),
    (dict(nd=0), hs.HS_ERR_INVALID_ARG),
    (dict(maxlen=0), hs.HS_ERR_INVALID_ARG),
    (dict(H=0), hs.HS_ERR_UNSUPPORTED),
    (dict(H=129), hs.HS_ERR_UNSUPPORTED),
    (dict(dk=2048), hs.HS_ERR_UNSUPPORTED),
    (dict(dt=5), hs.HS_ERR_UNSUPPORTED),
    (dict(qhs=100), hs.HS_ERR_INVALID_ARG),
    (dict(qrs=576), hs.HS_ERR_INVALID_ARG),
    (dict(krs=5), hs.HS_ERR_INVALID_ARG),
    (dict(B=48), hs.HS_ERR_UNSUPPORTED),
    (dict(lse=None), hs.HS_ERR_INVALID_ARG),
    (dict(nbs=1), hs.HS_ERR_INVALID_ARG),
    (dict(scale=float("nan")), hs.HS_ERR_INVALID_ARG),
])
def test_block_score_rejects_bad_arguments(kw, code):
    assert _score(**kw) == code
    assert hs.lib().hs_last_error()  # a message was recorded


def test_empty_input_is_a_no_op():
    # zero tokens: valid, nothing launched (no GPU needed)
    assert _score(T=0, nd=0, maxlen=0) == hs.HS_OK


def test_select_rejects_bad_arguments():
    L = hs.lib()
    p = ctypes.c_void_p(1)
    assert L.hs_select_topk(p, 4, p, 1, 100, 100, 64, 0, p, None) == hs.HS_ERR_UNSUPPORTED
    assert L.hs_select_topk(p, 4, p, 1, 100, 100, 64, 257, p, None) == hs.HS_ERR_UNSUPPORTED
    assert L.hs_select_topk(p, 1, p, 1, 100, 100, 64, 4, p, None) == hs.HS_ERR_INVALID_ARG
    assert L.hs_select_topk(None, 4, p, 1, 100, 100, 64, 4, p, None) == hs.HS_ERR_INVALID_ARG
    assert L.hs_select_topk(p, 4, p, 1, 100, 100, 20, 4, p, None) == hs.HS_ERR_UNSUPPORTED


def test_attention_rejects_bad_arguments():
    L = hs.lib()
    p = ctypes.c_void_p(1)
    args = [p, 64 * 576, 576, p, 576, p, 512, p, 1, 100, 100, 64, 576, 512, hs.HS_BF16, 0.0]
    # sparse: topk 0, NULL idx, bad block, bad v stride, NULL out
    assert L.hs_sparse_mqa_fwd(*args, p, 0, 64, None, p, p, None) == hs.HS_ERR_UNSUPPORTED
    assert L.hs_sparse_mqa_fwd(*args, None, 4, 64, None, p, p, None) == hs.HS_ERR_INVALID_ARG
    assert L.hs_sparse_mqa_fwd(*args, p, 4, 8, None, p, p, None) == hs.HS_ERR_UNSUPPORTED
    bad_v = list(args)
    bad_v[6] = 100
    assert L.hs_sparse_mqa_fwd(*bad_v, p, 4, 64, None, p, p, None) == hs.HS_ERR_INVALID_ARG
    assert L.hs_sparse_mqa_fwd(*args, p, 4, 64, None, None, p, None) == hs.HS_ERR_INVALID_ARG
    # swa: window 0, dv 0
    assert L.hs_swa_mqa_fwd(*args, 0, None, p, p, None) == hs.HS_ERR_INVALID_ARG
    no_dv = list(args)
    no_dv[13] = 0
    assert L.hs_swa_mqa_fwd(*no_dv, 16, None, p, p, None) == hs.HS_ERR_UNSUPPORTED



def test_backward_rejects_bad_arguments():
    L = hs.lib()
    p = ctypes.c_void_p(1)
    ws = ctypes.c_void_p(256)  # 16-byte aligned stand-in
    T, H = 100, 64
    need = L.hs_workspace_size(hs.HS_OP_SPARSE_MQA_BWD, T, 1, 100, H, 576, 512, hs.HS_BF16, 64)
    # delta / sink terms (8 T H, to 256 bytes), then the dk / dv pass's fp32
    # partial sums for its query ranges (ranges of >= 512 queries, <= 8)
    rlen = max(512, -(-T // 8))
    nrange = -(-T // rlen)
    assert need == (8 * T * H + 255) // 256 * 256 + nrange * T * (576 + 512) * 4
    assert L.hs_workspace_size(hs.HS_OP_SWA_MQA_BWD, T, 1, 100, H, 576, 512, hs.HS_BF16, 64) == need
    big = L.hs_workspace_size(hs.HS_OP_SPARSE_MQA_BWD, 65536, 1, 65536, H, 576, 512, hs.HS_BF16, 64)
    assert big == 8 * 65536 * H + 8 * 65536 * (576 + 512) * 4  # 8 ranges of 8192
    # CUDA-core shapes need only the delta / sink terms
    assert L.hs_workspace_size(hs.HS_OP_SPARSE_MQA_BWD, T, 1, 100, H, 576, 512, hs.HS_F32, 64) \
        == 8 * T * H
    assert L.hs_path(hs.HS_OP_SPARSE_MQA_BWD, hs.HS_BF16, H, 576, 512, 64) == hs.HS_PATH_MMA
    assert L.hs_path(hs.HS_OP_SWA_MQA_BWD, hs.HS_F32, H, 576, 512, 64) == hs.HS_PATH_SIMT
    assert L.hs_path(hs.HS_OP_SWA_MQA_BWD, hs.HS_BF16, 20, 80, 48, 64) == hs.HS_PATH_SIMT
    args = [p, 64 * 576, 576, p, 576, p, 512, p, 1, T, 100, H, 576, 512, hs.HS_BF16, 0.0]
    tail = [p, p, p, p, p, p, None]  # out, lse, dout, dq, dk, dv, dsink
    # sparse: bad topk / idx / block, missing gradient outputs, workspace
    assert L.hs_sparse_mqa_bwd(*args, p, 0, 64, None, *tail, ws, need, None) == hs.HS_ERR_UNSUPPORTED
    assert L.hs_sparse_mqa_bwd(*args, None, 4, 64, None, *tail, ws, need, None) == hs.HS_ERR_INVALID_ARG
    assert L.hs_sparse_mqa_bwd(*args, p, 4, 8, None, *tail, ws, need, None) == hs.HS_ERR_UNSUPPORTED
    no_dq = list(tail)
    no_dq[3] = None
    assert L.hs_sparse_mqa_bwd(*args, p, 4, 64, None, *no_dq, ws, need, None) == hs.HS_ERR_INVALID_ARG
    no_dout = list(tail)
    no_dout[2] = None
    assert L.hs_sparse_mqa_bwd(*args, p, 4, 64, None, *no_dout, ws, need, None) == hs.HS_ERR_INVALID_ARG
    assert L.hs_sparse_mqa_bwd(*args, p, 4, 64, None, *tail, None, need, None) == hs.HS_ERR_WORKSPACE
    assert L.hs_sparse_mqa_bwd(*args, p, 4, 64, None, *tail, ws, need - 1, None) == hs.HS_ERR_WORKSPACE
    odd = ctypes.c_void_p(258)
    assert L.hs_sparse_mqa_bwd(*args, p, 4, 64, None, *tail, odd, need, None) == hs.HS_ERR_INVALID_ARG
    # swa: window 0, short workspace
    assert L.hs_swa_mqa_bwd(*args, 0, None, *tail, ws, need, None) == hs.HS_ERR_INVALID_ARG
    assert L.hs_swa_mqa_bwd(*args, 16, None, *tail, ws, 0, None) == hs.HS_ERR_WORKSPACE
    # no tokens: nothing to do, no workspace needed
    empty = list(args)
    empty[9] = 0
    assert L.hs_swa_mqa_bwd(*empty, 16, None, *tail, None, 0, None) == hs.HS_OK

def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(4, 2, 8)
    k = torch.zeros(4, 8)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    with pytest.raises(ValueError):
        hs.hs_block_score(q, k, cu, 4, 16)


def test_selftest_rejects_bad_limit():
    L = hs.lib()
    assert L.hs_selftest_wait(0, None) == hs.HS_ERR_INVALID_ARG
    assert L.hs_selftest_wait(10**10, None) == hs.HS_ERR_INVALID_ARG


def test_full_layer_rejects_bad_arguments():
    L = hs.lib()
    p = ctypes.c_void_p(256)
    T, H = 100, 64
    ws = L.hs_workspace_size(hs.HS_OP_BLOCK_SCORE_ATTN, T, 1, 100, H, 576, 512, hs.HS_BF16, 64)
    # covers the fused kernel's scratch (2 rows of [NBmax, H] fp32 per CTA)
    # and step 1's kernel, which runs when the fused one is not eligible
    assert ws >= min(T, 148) * 2 * 2 * H * 4
    assert ws == L.hs_workspace_size(hs.HS_OP_BLOCK_SCORE, T, 1, 100, H, 576, 0, hs.HS_BF16, 64)
    assert L.hs_workspace_size(hs.HS_OP_BLOCK_SCORE_ATTN, T, 1, 100, 4, 64, 48, hs.HS_F32, 16) == 0
    assert L.hs_path(hs.HS_OP_BLOCK_SCORE_ATTN, hs.HS_BF16, H, 576, 512, 64) == hs.HS_PATH_TCGEN05
    assert L.hs_path(hs.HS_OP_BLOCK_SCORE_ATTN, hs.HS_F32, H, 576, 512, 64) == hs.HS_PATH_SIMT
    args = [p, 64 * 576, 576, p, 576, p, 512, p, 1, T, 100, H, 576, 512, hs.HS_BF16, 0.0]
    # block size, missing outputs, nb_stride below NBmax, missing v
    assert L.hs_block_score_attn_fwd(*args, 8, p, p, p, 2, None, p, ws, None) == hs.HS_ERR_UNSUPPORTED
    assert L.hs_block_score_attn_fwd(*args, 64, None, p, p, 2, None, p, ws, None) == hs.HS_ERR_INVALID_ARG
    assert L.hs_block_score_attn_fwd(*args, 64, p, p, None, 2, None, p, ws, None) == hs.HS_ERR_INVALID_ARG
    assert L.hs_block_score_attn_fwd(*args, 64, p, p, p, 1, None, p, ws, None) == hs.HS_ERR_INVALID_ARG
    no_v = list(args)
    no_v[5] = None
    assert L.hs_block_score_attn_fwd(*no_v, 64, p, p, p, 2, None, p, ws, None) == hs.HS_ERR_INVALID_ARG
    # no tokens: nothing to do
    empty = list(args)
    empty[9] = 0
    assert L.hs_block_score_attn_fwd(*empty, 64, p, p, p, 2, None, None, 0, None) == hs.HS_OK


def test_swa_layer_rejects_bad_arguments():
    L = hs.lib()
    p = ctypes.c_void_p(256)
    T, H = 100, 64
    assert L.hs_path(hs.HS_OP_SWA_LAYER, hs.HS_BF16, H, 576, 512, 64) == hs.HS_PATH_TCGEN05
    assert L.hs_workspace_size(hs.HS_OP_SWA_LAYER, T, 1, 100, H, 576, 512, hs.HS_BF16, 64) == 0
    head = [p, 64 * 576, 576, p, 576, p, 512]          # q, k, v
    shared = [p, 576, p, 512]                          # k_shared, v_shared
    common = [p, 1, T, 100, H, 576, 512, hs.HS_BF16, 0.0]
    def call(head=head, shared=shared, window=64, idx=p, topk=4, B=64, outs=(p, p, p)):
        return L.hs_swa_layer_fwd(*head, *shared, *common, window, None, idx, topk, B, None,
                                  None, None, *outs, None)
    assert call(window=0) == hs.HS_ERR_INVALID_ARG
    assert call(B=24) == hs.HS_ERR_UNSUPPORTED
    assert call(topk=0) == hs.HS_ERR_UNSUPPORTED
    assert call(idx=None) == hs.HS_ERR_INVALID_ARG
    assert call(shared=[None, 576, p, 512]) == hs.HS_ERR_INVALID_ARG
    assert call(shared=[p, 100, p, 512]) == hs.HS_ERR_INVALID_ARG
    assert call(head=[p, 64 * 576, 576, p, 576, None, 512]) == hs.HS_ERR_INVALID_ARG
    assert call(head=[p, 64 * 576, 576, p, 576, p, 500]) == hs.HS_ERR_INVALID_ARG
    assert call(outs=(p, None, p)) == hs.HS_ERR_INVALID_ARG
    assert call(outs=(p, p, None)) == hs.HS_ERR_INVALID_ARG


def test_package_version_matches_library():
    import block_sparse_mqa_b200 as pkg
    v = hs.lib().hs_version()
    assert pkg.__version__.split()[0] == "%d.%d.%d" % (v // 10000, v // 100 % 100, v % 100)


def test_last_path_is_minus_one_before_any_compute_call():
    # a rejected call does not change it; no call in this CPU process launches
    assert _score(B=48) == hs.HS_ERR_UNSUPPORTED
    assert hs.last_path() == -1


def _static(**kw):
    a = dict(q=1, qrs=64 * 576, qhs=576, k=1, krs=576, cu=1, nd=1, T=128, maxlen=128, H=64,
             dk=576, dt=hs.HS_BF16, scale=0.0, B=64, lse=1, bs=1, nbs=2, blse=NULL)
    a.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return hs.lib().hs_block_score_static(v(a["q"]), a["qrs"], a["qhs"], v(a["k"]), a["krs"],
                                          v(a["cu"]), a["nd"], a["T"], a["maxlen"], a["H"],
                                          a["dk"], a["dt"], a["scale"], a["B"], v(a["lse"]),
                                          v(a["bs"]), a["nbs"], v(a["blse"]), None)


@pytest.mark.parametrize("kw,code", [
    (dict(maxlen=-5), hs.HS_ERR_INVALID_ARG),   # must not wrap into a huge scratch size
    (dict(maxlen=0), hs.HS_ERR_INVALID_ARG),
    (dict(B=48), hs.HS_ERR_UNSUPPORTED),
    (dict(q=None), hs.HS_ERR_INVALID_ARG),
    (dict(nbs=1), hs.HS_ERR_INVALID_ARG),
    (dict(T=100000, maxlen=100000, nbs=1563), hs.HS_ERR_WORKSPACE),
])
def test_static_block_score_validates_before_sizing(kw, code):
    # arguments are checked on the host before the scratch size and before
    # any CUDA call, so none of these touches a device
    assert _static(**kw) == code
    assert hs.lib().hs_last_error()


def test_static_block_score_empty_input_is_a_no_op():
    assert _static(T=0, nd=0, maxlen=0) == hs.HS_OK
