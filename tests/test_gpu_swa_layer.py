"""GPU parity of the HySparse SWA layer (hs_swa_layer_fwd: window branch over
the layer's own KV plus the sparse branch over the full layer's shared KV,
gated sum) against the float64 oracle (``oracle.hysparse.swa_layer_fwd``).

The block lists of the sparse branch come from the oracle's own scoring of
the full layer's queries over the shared keys (uploaded for the GPU); rows
outside a sample keep GPU-selected lists and their outputs are not compared.
Tolerances are those of tests/parity.py (out 2e-2 max / 5e-3 relative
Frobenius, lse 1e-3).
"""

import numpy as np
import pytest
import torch

import oracle.hysparse as O
from block_sparse_mqa_b200 import hs, synth, workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda"


class Layer:
    """The SWA layer's q, own k / v and sink; the full layer's q, k / v and
    sink (its k / v are the shared KV); per-(token, head) gates."""

    def __init__(self, docs, H, dk, dv, dtype, seed=0, gates="random", alias_shared=False):
        T = sum(docs)
        own = synth.make_inputs(T, H, dk, dv, dtype=dtype, seed=seed, device=DEV,
                                doc_lengths=docs)
        full = synth.make_inputs(T, H, dk, dv, dtype=dtype, seed=seed + 50, device=DEV,
                                 doc_lengths=docs)
        self.q, self.k, self.v, self.sink_swa = own.q, own.k, own.v, own.sink
        self.qf, self.ks, self.sink_sparse = full.q, full.k, full.sink
        self.vs = full.k[:, :dv] if alias_shared else full.v
        self.cu, self.max_seqlen, self.T, self.H = own.cu_seqlens, own.max_seqlen, T, H
        g = torch.Generator(device=DEV)
        g.manual_seed(seed + 77)
        if gates == "random":
            self.gw = torch.rand((T, H), generator=g, device=DEV)
            self.gs = torch.rand((T, H), generator=g, device=DEV)
        elif gates == "none":
            self.gw = self.gs = None
        else:  # "swa_only"
            self.gw = torch.ones((T, H), device=DEV)
            self.gs = torch.zeros((T, H), device=DEV)


def _np(t):
    return None if t is None else t.detach().float().cpu().double().numpy()


def run_layer(L, B, K, W, rows=None, sinks=True):
    cu = L.cu.cpu().tolist()
    T = L.T
    rr = np.arange(T) if rows is None else np.asarray(rows)
    big = rows is not None and L.q.numel() > (1 << 27)

    def host_q(q):
        if not big:
            return _np(q)
        qs = _np(q[torch.as_tensor(rr, device=DEV)])
        return O.RowSubset({int(t): qs[i] for i, t in enumerate(rr)}, q.shape)

    q, qf = host_q(L.q), host_q(L.qf)
    k, v, ks, vs = _np(L.k), _np(L.v), _np(L.ks), _np(L.vs)
    # the full layer's block lists from the oracle for the compared rows
    ref_idx = O.select_topk(O.block_score(qf, ks, cu, B, rows=rr)["block_score"], cu, B, K,
                            rows=rr, total_tokens=T)
    if rows is None:
        idx = torch.as_tensor(np.ascontiguousarray(ref_idx, dtype=np.int32), device=DEV)
    else:  # other rows: the GPU's own selection (their outputs are ignored)
        _, bs, _ = hs.hs_block_score(L.qf, L.ks, L.cu, L.max_seqlen, B)
        idx = hs.hs_select_topk(bs, L.cu, L.max_seqlen, B, K)
        idx[torch.as_tensor(rr, device=DEV)] = torch.as_tensor(
            np.ascontiguousarray(ref_idx, dtype=np.int32), device=DEV)
    s1 = L.sink_swa if sinks else None
    s2 = L.sink_sparse if sinks else None
    out, lw, ls = hs.hs_swa_layer_fwd(L.q, L.k, L.v, L.ks, L.vs, idx, L.cu, L.max_seqlen, W, B,
                                      s1, s2, L.gw, L.gs)
    torch.cuda.synchronize()
    hs.poll_status()
    ref = O.swa_layer_fwd(q, k, v, ks, vs, ref_idx, cu, W, B, _np(s1), _np(s2), _np(L.gw),
                          _np(L.gs), rows=rr)
    rows_t = torch.as_tensor(rr, device=DEV)
    P.check_out(out[rows_t], ref["out"], "swa layer out")
    P.check_lse(lw[rows_t], ref["lse_swa"], "swa layer lse_swa")
    P.check_lse(ls[rows_t], ref["lse_sparse"], "swa layer lse_sparse")
    return out, lw, ls


def test_tiny_fp32_on_cuda_cores():
    L = Layer([256], 4, 64, 48, torch.float32, seed=0)
    assert hs.path(hs.HS_OP_SWA_LAYER, torch.float32, 4, 64, 48, 16) == hs.HS_PATH_SIMT
    run_layer(L, 16, 4, 32)


@pytest.mark.parametrize("gates", ["random", "none", "swa_only"])
def test_mla_shape_packed(gates):
    L = Layer([130, 64, 1, 257], 64, 576, 512, torch.bfloat16, seed=1, gates=gates)
    assert hs.path(hs.HS_OP_SWA_LAYER, torch.bfloat16, 64, 576, 512, 64) == hs.HS_PATH_TCGEN05
    run_layer(L, 64, 4, 100)


@pytest.mark.parametrize("dk,dv,B,K,W", [(512, 512, 32, 6, 300), (576, 448, 128, 3, 129),
                                         (128, 64, 16, 5, 1)])
def test_shape_and_block_variants(dk, dv, B, K, W):
    L = Layer([300, 37, 180], 64, dk, dv, torch.bfloat16, seed=2)
    run_layer(L, B, K, W)


def test_shared_v_aliases_shared_k_and_no_sinks():
    L = Layer([200, 133], 64, 576, 512, torch.bfloat16, seed=3, alias_shared=True)
    assert L.vs.stride(0) == 576
    run_layer(L, 64, 4, 64, sinks=False)


def test_zero_length_documents():
    L = Layer([0, 130, 0, 0, 257, 0], 64, 576, 512, torch.bfloat16, seed=9)
    run_layer(L, 64, 4, 100)


def test_forced_cuda_cores_agree():
    L = Layer([150, 90], 64, 576, 512, torch.bfloat16, seed=4)
    a = run_layer(L, 64, 4, 80)
    hs.set_force_simt(True)
    try:
        b = run_layer(L, 64, 4, 80)
    finally:
        hs.set_force_simt(False)
    P.check_out(a[0], b[0].cpu().double().numpy(), "tensor cores vs CUDA cores")


def test_main_workload_sampled():
    wl = workloads.MAIN
    L = Layer(wl.docs(), wl.num_heads, wl.dk, wl.dv, wl.dtype, seed=0)
    rows = synth.sample_rows(L.cu.cpu(), 24, 0)
    run_layer(L, wl.block_size, wl.topk, wl.window, rows=rows)


@pytest.mark.slow
def test_packed_workload_sampled():
    wl = workloads.PACKED
    L = Layer(wl.docs(), wl.num_heads, wl.dk, wl.dv, wl.dtype, seed=0)
    rows = synth.sample_rows(L.cu.cpu(), 6, 0)
    run_layer(L, wl.block_size, wl.topk, wl.window, rows=rows)


def test_empty_input_and_rejections():
    L = Layer([64], 64, 576, 512, torch.bfloat16, seed=8)
    idx = torch.zeros((64, 4), device=DEV, dtype=torch.int32)
    with pytest.raises(hs.HSError) as e:  # window < 1
        hs.hs_swa_layer_fwd(L.q, L.k, L.v, L.ks, L.vs, idx, L.cu, L.max_seqlen, 0, 64)
    assert e.value.status == hs.HS_ERR_INVALID_ARG
    with pytest.raises(ValueError):  # gates of the wrong shape
        hs.hs_swa_layer_fwd(L.q, L.k, L.v, L.ks, L.vs, idx, L.cu, L.max_seqlen, 16, 64,
                            gate_swa=torch.ones((64, 63), device=DEV))
