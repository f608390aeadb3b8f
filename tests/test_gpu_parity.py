"""GPU parity: every step of the CUDA path against the float64 CPU oracle on
the same seeded inputs, through the C ABI (ctypes binding).

Small cases compare every output element; the full-size workloads compare a
seeded sample of query rows (the oracle computes those rows one by one).
Tolerances are in tests/parity.py.
"""

import numpy as np
import pytest
import torch

import oracle.hysparse as O
from block_sparse_mqa_b200 import hs, synth, workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _gpu_inputs(T, H, dk, dv, dtype, docs, seed=0, sink_std=1.0):
    return synth.make_inputs(T, H, dk, dv, dtype=dtype, seed=seed, device=DEV, doc_lengths=docs,
                             sink_std=sink_std)


def _host(inp, rows=None):
    f = lambda t: t.detach().cpu().double().numpy()
    if rows is not None and inp.q.numel() > (1 << 27):  # only the sampled q rows
        rr = torch.as_tensor(np.asarray(rows), device=inp.q.device)
        qs = f(inp.q[rr])
        q = O.RowSubset({int(t): qs[i] for i, t in enumerate(rows)}, inp.q.shape)
    else:
        q = f(inp.q)
    return q, f(inp.k), f(inp.v), f(inp.sink), inp.cu_seqlens.cpu().tolist()


def _expect_path(op, inp, B):
    return hs.path(op, inp.q.dtype, inp.q.shape[1], inp.q.shape[2], inp.v.shape[1], B)


def run_and_check(inp, B, K, W, rows=None, sink=True, scale=0.0, v=None, check_paths=None):
    """Run the four steps on the GPU and compare each against the oracle.
    Stages are isolated without feeding GPU results to the oracle: the GPU
    re-runs selection on the oracle's scores and sparse attention on the
    oracle's index sets; the end-to-end index sets are compared too."""
    q, k, vv, s, cu = _host(inp, rows)
    v_dev = inp.v if v is None else v
    if v is not None:
        vv = v.detach().cpu().double().numpy()
    sink_dev = inp.sink if sink else None
    sink_np = s if sink else None
    T = inp.total_tokens
    rr = np.arange(T) if rows is None else np.asarray(rows)
    sc = None if scale == 0.0 else scale

    ran = {}  # kernel family each call actually launched (hs_last_path)
    lse1, bs, blse = hs.hs_block_score(inp.q, inp.k, inp.cu_seqlens, inp.max_seqlen, B, scale,
                                       want_block_lse=rows is None)
    ran["score"] = hs.last_path()
    idx = hs.hs_select_topk(bs, inp.cu_seqlens, inp.max_seqlen, B, K)
    out, lse = hs.hs_sparse_mqa_fwd(inp.q, inp.k, v_dev, idx, inp.cu_seqlens, inp.max_seqlen, B,
                                    sink_dev, scale)
    ran["sparse"] = hs.last_path()
    wout, wlse = hs.hs_swa_mqa_fwd(inp.q, inp.k, v_dev, inp.cu_seqlens, inp.max_seqlen, W,
                                   sink_dev, scale)
    ran["swa"] = hs.last_path()
    torch.cuda.synchronize()
    hs.poll_status()

    rows_t = torch.as_tensor(rr, device=DEV)
    ref1 = O.block_score(q, k, cu, B, scale=sc, rows=rr)
    nb = ref1["block_score"].shape[1]
    P.check_lse(lse1[rows_t], ref1["lse"], "score lse")
    P.check_scores(bs[rows_t], ref1["block_score"])
    if blse is not None:
        P.check_lse(blse[rows_t][:, :, :nb], ref1["block_lse"], "block_lse")
    # select, bit-exact: the GPU selects on the oracle's scores rounded to
    # fp32 on the host (rows outside the sample hold zeros and are ignored),
    # and the oracle selects on the same fp32 values
    nbs = bs.shape[1]
    bs32 = np.zeros((len(rr), nbs), dtype=np.float32)
    bs32[:, :nb] = ref1["block_score"].astype(np.float32)
    bs_in = torch.zeros((T, nbs), device=DEV, dtype=torch.float32)
    bs_in[rows_t] = torch.as_tensor(bs32, device=DEV)
    idx_on_ref = hs.hs_select_topk(bs_in, inp.cu_seqlens, inp.max_seqlen, B, K)
    ref_idx32 = O.select_topk(bs32[:, :nb].astype(np.float64), cu, B, K, rows=rr, total_tokens=T)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx_on_ref[rows_t].cpu().numpy(), ref_idx32)
    # the end-to-end GPU index sets against the oracle's (near-tie rule)
    idx_rows = idx[rows_t].cpu().numpy()
    ref_idx = O.select_topk(ref1["block_score"], cu, B, K, rows=rr, total_tokens=T)
    P.check_topk(idx_rows, ref_idx, ref1["block_score"], P.bq_rows(cu, rr, B), K)
    # sparse attention on the oracle's index sets (uploaded for the sampled
    # rows; the other rows keep the GPU's own, their outputs are ignored)
    idx_mix = idx.clone()
    idx_mix[rows_t] = torch.as_tensor(np.ascontiguousarray(ref_idx, dtype=np.int32), device=DEV)
    out_r, lse_r = hs.hs_sparse_mqa_fwd(inp.q, inp.k, v_dev, idx_mix, inp.cu_seqlens,
                                        inp.max_seqlen, B, sink_dev, scale)
    torch.cuda.synchronize()
    hs.poll_status()
    ref3 = O.sparse_mqa_fwd(q, k, vv, ref_idx, cu, B, sink=sink_np, scale=sc, rows=rr)
    P.check_out(out_r[rows_t], ref3["out"], "sparse out")
    P.check_lse(lse_r[rows_t], ref3["lse"], "sparse lse")
    ref4 = O.swa_mqa_fwd(q, k, vv, cu, W, sink=sink_np, scale=sc, rows=rr)
    P.check_out(wout[rows_t], ref4["out"], "swa out")
    P.check_lse(wlse[rows_t], ref4["lse"], "swa lse")
    return {"idx": idx, "out": out, "lse": lse, "swa_out": wout, "swa_lse": wlse, "bs": bs,
            "lse1": lse1, "ran": ran}


# ---------------------------------------------------------------------------
# small cases, every element
# ---------------------------------------------------------------------------

def test_tiny_fp32_workload():
    wl = workloads.TINY
    inp = _gpu_inputs(wl.total_tokens, wl.num_heads, wl.dk, wl.dv, wl.dtype, wl.docs())
    for op in (hs.HS_OP_BLOCK_SCORE, hs.HS_OP_SPARSE_MQA, hs.HS_OP_SWA_MQA):
        assert _expect_path(op, inp, wl.block_size) == hs.HS_PATH_SIMT
    run_and_check(inp, wl.block_size, wl.topk, wl.window)


@pytest.mark.parametrize("docs", [[452], [130, 64, 1, 257], [63, 65, 200, 124]])
def test_mla_shape_small_packed(docs):
    T = sum(docs)
    inp = _gpu_inputs(T, 64, 576, 512, torch.bfloat16, docs, seed=1)
    run_and_check(inp, 64, 4, 100)


@pytest.mark.parametrize("B,K,W", [(16, 3, 1), (32, 2, 700), (128, 5, 129), (64, 1, 64)])
def test_block_window_variants(B, K, W):
    docs = [300, 37, 180]
    inp = _gpu_inputs(sum(docs), 64, 576, 512, torch.bfloat16, docs, seed=2)
    run_and_check(inp, B, K, W)


@pytest.mark.parametrize("B,docs", [(16, [1000]), (32, [1300, 200])])
def test_many_blocks_per_row(B, docs):
    """More than 32 blocks per row with several query tiles per CTA: the
    epilogue's block batches and the next tile's workspace writes overlap."""
    inp = _gpu_inputs(sum(docs), 64, 576, 512, torch.bfloat16, docs, seed=11)
    run_and_check(inp, B, 6, 300)


@pytest.mark.parametrize("H,dk,dv", [(32, 576, 512), (128, 192, 128)])
def test_block_score_other_head_counts(H, dk, dv):
    docs = [400, 150]
    inp = _gpu_inputs(sum(docs), H, dk, dv, torch.bfloat16, docs, seed=12)
    assert hs.path(hs.HS_OP_BLOCK_SCORE, torch.bfloat16, H, dk, dv, 64) == hs.HS_PATH_TCGEN05
    run_and_check(inp, 64, 4, 100)


def test_no_sink_and_large_sink():
    docs = [200, 77]
    inp = _gpu_inputs(sum(docs), 64, 576, 512, torch.bfloat16, docs, seed=3)
    run_and_check(inp, 64, 3, 90, sink=False)
    inp.sink.fill_(8.0)
    run_and_check(inp, 64, 3, 90, sink=True)


def test_v_aliases_latent_part_of_k():
    docs = [260]
    inp = _gpu_inputs(sum(docs), 64, 576, 512, torch.bfloat16, docs, seed=4)
    v_alias = inp.k[:, :512]  # absorbed-MLA: value = latent region of the key row
    assert v_alias.data_ptr() == inp.k.data_ptr()
    res = run_and_check(inp, 64, 3, 128, v=v_alias)
    assert res["ran"] == {"score": hs.HS_PATH_TCGEN05, "sparse": hs.HS_PATH_TCGEN05,
                          "swa": hs.HS_PATH_TCGEN05}


def test_strided_q_and_explicit_scale():
    docs = [150, 90]
    T = sum(docs)
    base = _gpu_inputs(T, 64, 576, 512, torch.bfloat16, docs, seed=5)
    big = torch.zeros((T, 66, 640), device=DEV, dtype=torch.bfloat16)
    big[:, :64, :576] = base.q
    base.q = big[:, :64, :576]
    assert base.q.stride() == (66 * 640, 640, 1)
    res = run_and_check(base, 64, 3, 70, scale=0.03)
    assert set(res["ran"].values()) == {hs.HS_PATH_TCGEN05}


def test_last_path_reports_a_stride_fallback():
    """A q head stride that is not a multiple of 8 elements cannot be a TMA
    operand, so those calls run on the CUDA-core kernels although hs_path
    (which sees only the shape) names the tensor-core path; hs_last_path
    reports what ran, and the results still match the oracle."""
    docs = [150, 90]
    T = sum(docs)
    base = _gpu_inputs(T, 64, 576, 512, torch.bfloat16, docs, seed=5)
    big = torch.zeros((T, 64, 580), device=DEV, dtype=torch.bfloat16)
    big[:, :, :576] = base.q
    base.q = big[:, :, :576]
    assert base.q.stride(1) % 8 != 0
    assert _expect_path(hs.HS_OP_SPARSE_MQA, base, 64) == hs.HS_PATH_TCGEN05
    res = run_and_check(base, 64, 3, 70)
    assert res["ran"] == {"score": hs.HS_PATH_SIMT, "sparse": hs.HS_PATH_SIMT,
                          "swa": hs.HS_PATH_SIMT}
    hs.hs_select_topk(res["bs"], base.cu_seqlens, base.max_seqlen, 64, 3)
    assert hs.last_path() == hs.HS_PATH_SIMT  # selection is never a contraction


def test_other_head_counts_and_dims():
    for H, dk, dv in ((4, 64, 48), (16, 192, 128), (64, 192, 128), (8, 40, 24)):
        docs = [150, 61]
        inp = _gpu_inputs(sum(docs), H, dk, dv, torch.bfloat16, docs, seed=6)
        run_and_check(inp, 16, 4, 33)



@pytest.mark.parametrize("dk,dv", [(512, 512), (576, 448), (448, 256), (256, 192), (128, 64),
                                   (64, 128)])
def test_shape_variants_on_tensor_cores(dk, dv):
    """Dk = 512 (no RoPE chunk, "FlashMLA sparse kernel constraints": d_qk in
    {512, 576}), Dv below 512 natively (kv_lora_rank < 512) and other widths
    that are multiples of 64: both block scoring and attention stay on the
    tensor-core path."""
    docs = [260, 71, 130]
    inp = _gpu_inputs(sum(docs), 64, dk, dv, torch.bfloat16, docs, seed=14)
    for op in (hs.HS_OP_BLOCK_SCORE, hs.HS_OP_SPARSE_MQA, hs.HS_OP_SWA_MQA):
        assert _expect_path(op, inp, 64) == hs.HS_PATH_TCGEN05, (op, dk, dv)
    run_and_check(inp, 64, 4, 100)

@pytest.mark.parametrize("dtype,H,dk,dv", [(torch.bfloat16, 64, 576, 512),
                                          (torch.float32, 4, 64, 48)])
def test_zero_length_documents(dtype, H, dk, dv):
    """cu_seqlens may repeat an offset (an empty document, e.g. padding);
    empty documents own no rows and no blocks, and block numbering restarts
    at each non-empty document."""
    docs = [0, 200, 0, 0, 133, 0]
    inp = _gpu_inputs(sum(docs), H, dk, dv, dtype, docs, seed=15)
    run_and_check(inp, 64 if H == 64 else 16, 4, 100)


def test_topk_at_maximum_covers_every_block():
    """topk = 256 (the largest accepted) selects every causal block of these
    documents, so block-sparse attention is dense causal attention, which the
    window kernel computes with a window longer than the documents (the
    oracle's invariant, here between the two GPU kernels)."""
    docs = [700, 90]
    inp = _gpu_inputs(sum(docs), 64, 576, 512, torch.bfloat16, docs, seed=16)
    res = run_and_check(inp, 16, 256, 1000)
    P.check_out(res["out"], P.np64(res["swa_out"]), "sparse (all blocks) vs window (all keys)")
    P.check_lse(res["lse"], P.np64(res["swa_lse"]), "sparse vs window lse")


@pytest.mark.parametrize("B,K,docs", [(64, 6, [700, 0, 420]), (16, 10, [400, 0, 300])])
def test_planted_block_order_selects_exactly(B, K, docs):
    """Structured inputs (synth.plant_block_order, gap 3 natural-log units
    per rank): the block order is planted, so the GPU's index sets must equal
    the selection rule's choice for that order exactly, with no near-tie
    excusal; every step still matches the oracle.  Documents stay under 27
    blocks so that no selected block's fp32 score underflows."""
    base = _gpu_inputs(sum(docs), 64, 576, 512, torch.bfloat16, docs, seed=17)
    inp, perms = synth.plant_block_order(base, B, gap=3.0, seed=17)
    res = run_and_check(inp, B, K, 100)
    expect = P.planted_selection(inp.cu_seqlens.cpu(), perms, B, K)
    np.testing.assert_array_equal(res["idx"].cpu().numpy(), expect)


def test_force_simt_agrees_with_default_path():
    docs = [333, 80]
    inp = _gpu_inputs(sum(docs), 64, 576, 512, torch.bfloat16, docs, seed=7)
    a = hs.hs_forward(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen, 64, 4, 100, inp.sink)
    hs.set_force_simt(True)
    try:
        b = hs.hs_forward(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen, 64, 4, 100, inp.sink)
    finally:
        hs.set_force_simt(False)
    torch.cuda.synchronize()
    np.testing.assert_allclose(a["block_score"].cpu(), b["block_score"].cpu(), rtol=2e-4, atol=1e-5)
    P.check_lse(a["sparse_lse"], P.np64(b["sparse_lse"]))
    P.check_out(a["swa_out"], P.np64(b["swa_out"]))


# ---------------------------------------------------------------------------
# device-detected errors
# ---------------------------------------------------------------------------

def test_invalid_index_reported():
    docs = [200]
    inp = _gpu_inputs(200, 64, 576, 512, torch.bfloat16, docs, seed=8)
    idx = torch.full((200, 2), -1, device=DEV, dtype=torch.int32)
    idx[:, 0] = torch.arange(200, device=DEV, dtype=torch.int32) // 64
    idx[5, 1] = 3  # block 3 is in the future of token 5
    hs.hs_sparse_mqa_fwd(inp.q, inp.k, inp.v, idx, inp.cu_seqlens, 200, 64, inp.sink)
    with pytest.raises(hs.HSError) as e:
        hs.poll_status()
    assert e.value.status == hs.HS_ERR_INVALID_INDEX
    hs.poll_status()  # cleared


def test_malformed_cu_seqlens_reported():
    inp = _gpu_inputs(128, 64, 576, 512, torch.bfloat16, [128], seed=9)
    bad = torch.tensor([0, 100, 128], device=DEV, dtype=torch.int32)
    # max_seqlen 64 is smaller than the first document: rows of it are skipped
    lse, bs, _ = hs.hs_block_score(inp.q, inp.k, bad, 64, 64)
    with pytest.raises(hs.HSError) as e:
        hs.poll_status()
    assert e.value.status == hs.HS_ERR_INVALID_ARG


# ---------------------------------------------------------------------------
# full-size workloads, sampled rows
# ---------------------------------------------------------------------------

def _sampled(wl, per_doc, seed=0):
    inp = _gpu_inputs(wl.total_tokens, wl.num_heads, wl.dk, wl.dv, wl.dtype, wl.docs(), seed=seed)
    rows = synth.sample_rows(inp.cu_seqlens.cpu(), per_doc, seed)
    return inp, rows


def test_main_workload_sampled():
    wl = workloads.MAIN
    inp, rows = _sampled(wl, 48)
    run_and_check(inp, wl.block_size, wl.topk, wl.window, rows=rows)


@pytest.mark.parametrize("wl", [workloads.NOROPE, workloads.NARROW_V], ids=lambda w: w.name)
def test_shape_variant_workloads_sampled(wl):
    inp, rows = _sampled(wl, 24)
    for op in (hs.HS_OP_BLOCK_SCORE, hs.HS_OP_SPARSE_MQA, hs.HS_OP_SWA_MQA):
        assert _expect_path(op, inp, wl.block_size) == hs.HS_PATH_TCGEN05
    run_and_check(inp, wl.block_size, wl.topk, wl.window, rows=rows)


@pytest.mark.slow
def test_packed_workload_sampled():
    wl = workloads.PACKED
    inp, rows = _sampled(wl, 12)
    run_and_check(inp, wl.block_size, wl.topk, wl.window, rows=rows)


@pytest.mark.slow
def test_long_context_workload_sampled():
    wl = workloads.LONG
    inp, rows = _sampled(wl, 16)
    run_and_check(inp, wl.block_size, wl.topk, wl.window, rows=rows)


@pytest.mark.slow
@pytest.mark.parametrize("topk", [8, 16, 32, 64])
def test_sweep_workload_sampled(topk):
    wl = workloads.sweep(topk)
    inp, rows = _sampled(wl, 5)
    run_and_check(inp, wl.block_size, wl.topk, wl.window, rows=rows)


@pytest.mark.slow
@pytest.mark.parametrize("window", [256, 1024, 4096])
def test_sweep_swa_layer_sampled(window):
    """The separate SWA-only layer of the sweep: Dk 192, Dv 128."""
    wl = workloads.sweep_swa(window)
    inp, rows = _sampled(wl, 6)
    assert hs.path(hs.HS_OP_SWA_MQA, wl.dtype, 64, 192, 128, 64) == hs.HS_PATH_TCGEN05
    q, k, vv, s, cu = _host(inp, rows)
    wout, wlse = hs.hs_swa_mqa_fwd(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen, window,
                                   inp.sink)
    torch.cuda.synchronize()
    hs.poll_status()
    rows_t = torch.as_tensor(rows, device=DEV)
    ref = O.swa_mqa_fwd(q, k, vv, cu, window, sink=s, rows=rows)
    P.check_out(wout[rows_t], ref["out"], "swa out")
    P.check_lse(wlse[rows_t], ref["lse"], "swa lse")
