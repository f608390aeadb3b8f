"""GPU parity of the attention backward (hs_sparse_mqa_bwd, hs_swa_mqa_bwd)
against the float64 oracle (``oracle.backward``) on the same seeded inputs.

Inputs flow one way: q, k, v, sink and dout come from the seeded generators;
the block lists come from the oracle's own selection and are uploaded for the
GPU; the GPU forward supplies out and lse to the GPU backward only.  The
oracle recomputes everything from the inputs.

Tolerances (on each gradient, relative to the oracle):

* fp32 inputs: ||gpu - ref||_F / ||ref||_F <= 1e-4 and max |gpu - ref| <=
  1e-3 * max |ref| (fp32 accumulation over at most a few thousand terms).
* bf16 inputs: 1e-2 and 5e-2.  The backward reads the forward's out, which
  is rounded to bf16 (relative error up to 2^-9); that error enters every
  ds_j through delta = <dout, out>, where ds_j = p_j (dp_j - delta) can
  cancel, so it is amplified by |delta| / |dp_j - delta| for some keys.  The
  bound on the Frobenius norm is the forward's out bound doubled.
"""

import numpy as np
import pytest
import torch

import oracle.backward as OB
import oracle.hysparse as O
from block_sparse_mqa_b200 import hs, synth, workloads

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = {torch.float32: (1e-4, 1e-3), torch.bfloat16: (1e-2, 5e-2)}


def _np(t):
    return t.detach().float().cpu().double().numpy()


def _dout(T, H, dv, dtype, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(1000 + seed)
    return torch.randn((T, H, dv), generator=g, device=DEV, dtype=torch.float32).to(dtype)


def check_grad(gpu, ref, dtype, what):
    fro_tol, max_tol = TOL[dtype]
    g = _np(gpu)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), what + ": non-finite"
    scale = max(float(np.abs(r).max()), 1e-30)
    fro = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
    mx = float(np.abs(g - r).max()) / scale
    assert fro <= fro_tol, "%s rel Frobenius err %.3e > %.1e" % (what, fro, fro_tol)
    assert mx <= max_tol, "%s max err %.3e of max|ref| > %.1e" % (what, mx, max_tol)
    return fro, mx


def run_backward(docs, H, dk, dv, dtype, kind, B=64, K=4, W=100, sink=True, seed=0, idx_edit=None):
    T = sum(docs)
    inp = synth.make_inputs(T, H, dk, dv, dtype=dtype, seed=seed, device=DEV, doc_lengths=docs)
    q, k, v, s = _np(inp.q), _np(inp.k), _np(inp.v), _np(inp.sink)
    cu = inp.cu_seqlens.cpu().tolist()
    sink_dev, sink_np = (inp.sink, s) if sink else (None, None)
    dout = _dout(T, H, dv, dtype, seed)
    if kind == "sparse":
        ref_idx = O.select_topk(O.block_score(q, k, cu, B)["block_score"], cu, B, K)
        if idx_edit is not None:
            ref_idx = idx_edit(ref_idx)
        idx = torch.as_tensor(np.ascontiguousarray(ref_idx, dtype=np.int32), device=DEV)
        out, lse = hs.hs_sparse_mqa_fwd(inp.q, inp.k, inp.v, idx, inp.cu_seqlens, inp.max_seqlen,
                                        B, sink_dev)
        g = hs.hs_sparse_mqa_bwd(inp.q, inp.k, inp.v, idx, inp.cu_seqlens, inp.max_seqlen, B,
                                 out, lse, dout, sink_dev)
        ref = OB.sparse_mqa_bwd(q, k, v, _np(dout), ref_idx, cu, B, sink=sink_np)
    else:
        out, lse = hs.hs_swa_mqa_fwd(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen, W,
                                     sink_dev)
        g = hs.hs_swa_mqa_bwd(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen, W, out, lse,
                              dout, sink_dev)
        ref = OB.swa_mqa_bwd(q, k, v, _np(dout), cu, W, sink=sink_np)
    torch.cuda.synchronize()
    hs.poll_status()
    for gpu, name in zip(g[:3], ("dq", "dk", "dv")):
        check_grad(gpu, ref[name], dtype, kind + " " + name)
    if sink:
        check_grad(g[3], ref["dsink"], dtype, kind + " dsink")
    else:
        assert g[3] is None
    return g


@pytest.mark.parametrize("sink", [True, False])
@pytest.mark.parametrize("kind", ["sparse", "swa"])
def test_backward_fp32_small(kind, sink):
    run_backward([97, 40, 1, 150], 4, 64, 48, torch.float32, kind, B=16, K=4, W=40, sink=sink)


@pytest.mark.parametrize("kind", ["sparse", "swa"])
def test_backward_mla_shape_packed(kind):
    run_backward([130, 64, 1, 257], 64, 576, 512, torch.bfloat16, kind, B=64, K=4, W=100, seed=1)


@pytest.mark.parametrize("B,K,W", [(16, 3, 1), (32, 2, 700), (128, 5, 129)])
def test_backward_block_and_window_variants(B, K, W):
    docs = [300, 37, 180]
    for kind in ("sparse", "swa"):
        run_backward(docs, 8, 128, 64, torch.bfloat16, kind, B=B, K=K, W=W, seed=2)


@pytest.mark.parametrize("B,K,W,dk,dv", [(16, 3, 1, 128, 64), (32, 2, 700, 192, 128),
                                         (128, 5, 129, 512, 448), (64, 4, 64, 64, 512)])
def test_backward_tensor_core_variants(B, K, W, dk, dv):
    """64 heads in bf16 take the tcgen05 passes (query-major dq over 128-key
    tiles, key-major dk/dv over 32-key tiles): block sizes whose blocks a
    32-key tile can straddle (three at B = 16), documents that start off the
    tile grids, Dk / Dv multiples of 64 down to a single 64-column chunk and
    a ragged last 128-row chunk (Dv = 448)."""
    docs = [300, 37, 180]
    for kind in ("sparse", "swa"):
        run_backward(docs, 64, dk, dv, torch.bfloat16, kind, B=B, K=K, W=W, seed=3)



def test_backward_paths_and_forced_cuda_cores():
    assert hs.path(hs.HS_OP_SPARSE_MQA_BWD, torch.bfloat16, 64, 576, 512, 64) == hs.HS_PATH_MMA
    assert hs.path(hs.HS_OP_SWA_MQA_BWD, torch.float32, 64, 576, 512, 64) == hs.HS_PATH_SIMT
    hs.set_force_simt(True)
    try:
        assert hs.path(hs.HS_OP_SPARSE_MQA_BWD, torch.bfloat16, 64, 576, 512, 64) == hs.HS_PATH_SIMT
        for kind in ("sparse", "swa"):
            run_backward([130, 64, 1, 257], 64, 576, 512, torch.bfloat16, kind, seed=1)
    finally:
        hs.set_force_simt(False)


def test_backward_with_v_aliasing_k():
    """v = k[:, :Dv] (the absorbed-MLA latent slice, a strided view of k): the
    call returns the gradients of its k and v arguments separately; the
    caller adds dv into the first Dv columns of dk."""
    docs = [200, 133]
    T, H, dk, dv = sum(docs), 64, 576, 512
    inp = synth.make_inputs(T, H, dk, dv, dtype=torch.bfloat16, seed=21, device=DEV,
                            doc_lengths=docs)
    v = inp.k[:, :dv]
    assert v.stride(0) == dk
    q, k, s = _np(inp.q), _np(inp.k), _np(inp.sink)
    cu = inp.cu_seqlens.cpu().tolist()
    dout = _dout(T, H, dv, torch.bfloat16, 21)
    ref_idx = O.select_topk(O.block_score(q, k, cu, 64)["block_score"], cu, 64, 4)
    idx = torch.as_tensor(np.ascontiguousarray(ref_idx, dtype=np.int32), device=DEV)
    out, lse = hs.hs_sparse_mqa_fwd(inp.q, inp.k, v, idx, inp.cu_seqlens, inp.max_seqlen, 64,
                                    inp.sink)
    g = hs.hs_sparse_mqa_bwd(inp.q, inp.k, v, idx, inp.cu_seqlens, inp.max_seqlen, 64, out, lse,
                             dout, inp.sink)
    torch.cuda.synchronize()
    hs.poll_status()
    ref = OB.sparse_mqa_bwd(q, k, k[:, :dv], _np(dout), ref_idx, cu, 64, sink=s)
    for gpu, name in zip(g, ("dq", "dk", "dv", "dsink")):
        check_grad(gpu, ref[name], torch.bfloat16, "aliased " + name)

@pytest.mark.parametrize("kind", ["sparse", "swa"])
def test_backward_zero_length_documents(kind):
    run_backward([0, 150, 0, 0, 97, 0], 64, 576, 512, torch.bfloat16, kind, seed=12)


def test_backward_other_dims():
    # Dk != Dv, not multiples of 64; several head groups with a partial last one
    run_backward([120, 88], 20, 80, 48, torch.float32, "sparse", B=16, K=3, seed=4)
    run_backward([120, 88], 20, 80, 48, torch.float32, "swa", W=33, seed=4)


def test_backward_rows_without_blocks():
    # rows whose idx holds no usable block attend to nothing: out = 0, only the
    # sink; their dq is 0 and they add nothing to dk / dv
    def edit(ix):
        ix = ix.copy()
        ix[5:40:3] = -1
        return ix
    g = run_backward([200], 4, 64, 48, torch.float32, "sparse", B=16, K=3, seed=5, idx_edit=edit)
    dq = g[0].cpu().numpy()
    assert np.all(dq[5:40:3] == 0.0)


def test_backward_is_deterministic():
    docs = [150, 90]
    T = sum(docs)
    inp = synth.make_inputs(T, 64, 576, 512, dtype=torch.bfloat16, seed=6, device=DEV,
                            doc_lengths=docs)
    dout = _dout(T, 64, 512, torch.bfloat16, 6)
    out, lse = hs.hs_swa_mqa_fwd(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen, 64, inp.sink)
    a = hs.hs_swa_mqa_bwd(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen, 64, out, lse,
                          dout, inp.sink)
    b = hs.hs_swa_mqa_bwd(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen, 64, out, lse,
                          dout, inp.sink)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.slow
@pytest.mark.parametrize("kind", ["sparse", "swa"])
def test_backward_main_workload(kind):
    wl = workloads.MAIN
    run_backward(wl.docs(), wl.num_heads, wl.dk, wl.dv, wl.dtype, kind, B=wl.block_size,
                 K=wl.topk, W=wl.window, seed=0)
