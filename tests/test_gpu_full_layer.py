"""GPU parity of the full layer's forward with step 1 fused in
(hs_block_score_attn_fwd) against the float64 oracle
(``oracle.hysparse.full_layer_fwd``) on the same seeded inputs.

Tolerances are those of tests/parity.py: out as the attention steps, lse and
block_lse to 1e-3 absolute, block_score to 1e-4 relative.  The top-k sets
chosen from the fused kernel's scores must equal the oracle's up to the
near-tie rule.
"""

import numpy as np
import pytest
import torch

import oracle.hysparse as O
from block_sparse_mqa_b200 import hs, synth, workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(docs, H, dk, dv, dtype, seed=0):
    return synth.make_inputs(sum(docs), H, dk, dv, dtype=dtype, seed=seed, device=DEV,
                             doc_lengths=docs)


def _host(inp, rows=None):
    f = lambda t: t.detach().cpu().double().numpy()
    if rows is not None and inp.q.numel() > (1 << 27):  # only the sampled q rows
        rr = torch.as_tensor(np.asarray(rows), device=inp.q.device)
        qs = f(inp.q[rr])
        q = O.RowSubset({int(t): qs[i] for i, t in enumerate(rows)}, inp.q.shape)
    else:
        q = f(inp.q)
    return q, f(inp.k), f(inp.v), inp.cu_seqlens.cpu().tolist()


def run_full(inp, B, rows=None, scale=0.0, want_blse=True, topk=4, nb_pad=0):
    q, k, v, cu = _host(inp, rows)
    T = inp.total_tokens
    rr = np.arange(T) if rows is None else np.asarray(rows)
    sc = None if scale == 0.0 else scale
    nb = hs.nbmax(inp.max_seqlen, B)
    H = inp.q.shape[1]
    # outputs with nb_pad extra columns holding a sentinel the call must not touch
    bs_buf = torch.full((T, nb + nb_pad), float("nan"), device=DEV)
    blse_buf = (torch.full((T, H, nb + nb_pad), float("nan"), device=DEV)
                if want_blse else None)
    out, lse, bs, blse = hs.hs_block_score_attn_fwd(
        inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen, B, scale,
        out_block_score=bs_buf, out_block_lse=blse_buf)
    torch.cuda.synchronize()
    hs.poll_status()
    if nb_pad:
        assert torch.isnan(bs[:, nb:]).all()
        if want_blse:
            assert torch.isnan(blse[:, :, nb:]).all()
    ref = O.full_layer_fwd(q, k, v, cu, B, scale=sc, rows=rr)
    rows_t = torch.as_tensor(rr, device=DEV)
    P.check_out(out[rows_t], ref["out"], "full out")
    P.check_lse(lse[rows_t], ref["lse"], "full lse")
    P.check_scores(bs[rows_t][:, :nb], ref["block_score"], "full block_score")
    if want_blse:
        P.check_lse(blse[rows_t][:, :, :nb], ref["block_lse"], "full block_lse")
    # top-k on the fused scores against the oracle's selection
    idx = hs.hs_select_topk(bs, inp.cu_seqlens, inp.max_seqlen, B, topk)
    torch.cuda.synchronize()
    ref_idx = O.select_topk(ref["block_score"], cu, B, topk, rows=rr, total_tokens=T)
    P.check_topk(idx[rows_t].cpu().numpy(), ref_idx, ref["block_score"], P.bq_rows(cu, rr, B),
                 topk)
    return out, lse, bs, blse


def test_tiny_fp32_on_cuda_cores():
    """fp32 runs the attention and the step-1 kernel one after the other."""
    inp = _inputs([256], 4, 64, 48, torch.float32, seed=0)
    assert hs.path(hs.HS_OP_BLOCK_SCORE_ATTN, torch.float32, 4, 64, 48, 16) == hs.HS_PATH_SIMT
    run_full(inp, 16, nb_pad=3)


@pytest.mark.parametrize("B", [32, 64, 128])
def test_mla_shape_packed_fused(B):
    """bf16, 64 heads, Dk 576 / Dv 512: the fused tcgen05 kernel; documents
    that start off the 128-key tile grid, a one-token document, ragged
    last blocks and tiles."""
    inp = _inputs([130, 64, 1, 257, 300], 64, 576, 512, torch.bfloat16, seed=1)
    assert hs.path(hs.HS_OP_BLOCK_SCORE_ATTN, torch.bfloat16, 64, 576, 512, B) == \
        hs.HS_PATH_TCGEN05
    run_full(inp, B, nb_pad=2)


def test_block16_runs_two_tensor_core_kernels():
    inp = _inputs([200, 77], 64, 576, 512, torch.bfloat16, seed=2)
    run_full(inp, 16)


@pytest.mark.parametrize("dk,dv", [(512, 512), (576, 448), (128, 64), (64, 128)])
def test_shape_variants_fused(dk, dv):
    inp = _inputs([190, 321], 64, dk, dv, torch.bfloat16, seed=3)
    run_full(inp, 64)


def test_zero_length_documents():
    inp = _inputs([0, 130, 0, 0, 257, 0], 64, 576, 512, torch.bfloat16, seed=8)
    run_full(inp, 64)


def test_forced_cuda_cores_agree():
    inp = _inputs([150, 90], 64, 576, 512, torch.bfloat16, seed=4)
    a = run_full(inp, 64)
    hs.set_force_simt(True)
    try:
        b = run_full(inp, 64)
    finally:
        hs.set_force_simt(False)
    np.testing.assert_allclose(a[2].cpu(), b[2].cpu(), rtol=2e-4, atol=1e-5)


def test_without_block_lse_and_explicit_scale():
    inp = _inputs([333], 64, 576, 512, torch.bfloat16, seed=5)
    run_full(inp, 64, want_blse=False, scale=0.05)


def test_matches_separate_step1_and_is_deterministic():
    """The fused scores equal step 1's kernel within the score tolerance, and
    two calls give identical bits."""
    inp = _inputs([400, 123], 64, 576, 512, torch.bfloat16, seed=6)
    o1, l1, s1, b1 = hs.hs_block_score_attn_fwd(inp.q, inp.k, inp.v, inp.cu_seqlens,
                                                inp.max_seqlen, 64, want_block_lse=True)
    o2, l2, s2, b2 = hs.hs_block_score_attn_fwd(inp.q, inp.k, inp.v, inp.cu_seqlens,
                                                inp.max_seqlen, 64, want_block_lse=True)
    lse_s, bs_s, _ = hs.hs_block_score(inp.q, inp.k, inp.cu_seqlens, inp.max_seqlen, 64)
    torch.cuda.synchronize()
    hs.poll_status()
    for x, y in ((o1, o2), (l1, l2), (s1, s2), (b1, b2)):
        assert torch.equal(x, y)
    P.check_scores(s1, bs_s.cpu().double().numpy(), "fused vs step 1")
    P.check_lse(l1, lse_s.cpu().double().numpy(), "fused lse vs step 1")


def test_main_workload_sampled():
    wl = workloads.MAIN
    inp = synth.make_inputs(wl.total_tokens, wl.num_heads, wl.dk, wl.dv, dtype=wl.dtype, seed=0,
                            device=DEV, doc_lengths=wl.docs())
    rows = synth.sample_rows(inp.cu_seqlens.cpu(), 32, 0)
    run_full(inp, wl.block_size, rows=rows, topk=wl.topk)


@pytest.mark.slow
def test_packed_workload_sampled():
    wl = workloads.PACKED
    inp = synth.make_inputs(wl.total_tokens, wl.num_heads, wl.dk, wl.dv, dtype=wl.dtype, seed=0,
                            device=DEV, doc_lengths=wl.docs())
    rows = synth.sample_rows(inp.cu_seqlens.cpu(), 8, 0)
    run_full(inp, wl.block_size, rows=rows, topk=wl.topk)


@pytest.mark.slow
def test_long_context_workload_sampled():
    """T = 65536 in one document: 1024 key blocks per row, the per-SM block
    scratch at its largest."""
    wl = workloads.LONG
    inp = synth.make_inputs(wl.total_tokens, wl.num_heads, wl.dk, wl.dv, dtype=wl.dtype, seed=0,
                            device=DEV, doc_lengths=wl.docs())
    rows = synth.sample_rows(inp.cu_seqlens.cpu(), 10, 0)
    run_full(inp, wl.block_size, rows=rows, topk=wl.topk, want_blse=False)


def test_short_workspace_is_refused():
    inp = _inputs([300], 64, 576, 512, torch.bfloat16, seed=7)
    need = hs.workspace_size(hs.HS_OP_BLOCK_SCORE_ATTN, 300, 1, inp.max_seqlen, 64, 576, 512,
                             torch.bfloat16, 64)
    assert need > 1024  # the fused kernel alone needs 2 x NBmax x 64 fp32 per SM
    ws = torch.empty(1024, device=DEV, dtype=torch.uint8)
    with pytest.raises(hs.HSError) as e:
        hs.hs_block_score_attn_fwd(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen, 64,
                                   workspace=ws)
    assert e.value.status == hs.HS_ERR_WORKSPACE
