"""Pins for the CPU oracle (no GPU).

Each test checks ``oracle.hysparse`` against something other than itself:
hand-derived closed forms (tests/golden/closed_form.json), a library routine
(torch float64 logsumexp / scaled_dot_product_attention), a pure-Python loop
restatement (``oracle.loops``), exhaustive search, or an invariant that the
definitions fix.  The definitions are those of "HySparse MQA sparse
attention (FA4 block scoring + SWA MQA + block-sparse DSA gather)",
PaddleFleet pull request 1470 ("Core" list, per-file table), with the sink
read as a softmax-denominator offset ("Support attn sink in fa3", pull
request 1415) and the full-coverage invariant of the "Unified sparse
attention API (dispatcher)" page (model-config key points).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.hysparse as O
from oracle import loops
from block_sparse_mqa_b200 import synth
from tests import parity as P

GOLD = os.path.join(os.path.dirname(__file__), "golden", "closed_form.json")


def _np(x):
    return x.detach().cpu().double().numpy()


def _inputs(T, H, dk, dv, docs=None, seed=0, dtype=torch.float32):
    inp = synth.make_inputs(T, H, dk, dv, dtype=dtype, seed=seed, doc_lengths=docs)
    return _np(inp.q), _np(inp.k), _np(inp.v), _np(inp.sink), inp.cu_seqlens.tolist()


def _none_to_inf(a):
    return np.array([[[(-math.inf if x is None else x) for x in r] for r in h] for h in a])


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def test_golden_example_a():
    ex = json.load(open(GOLD))["example_a"]
    q, k, v = (np.array(ex[n]) for n in ("q", "k", "v"))
    cu, sc, B = ex["cu_seqlens"], ex["scale"], ex["block_size"]
    sink = np.array(ex["sink"])
    e = ex["expect"]
    bs = O.block_score(q, k, cu, B, scale=sc)
    np.testing.assert_allclose(bs["lse"], e["lse"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(bs["block_score"], e["block_score"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(bs["block_lse"], _none_to_inf(e["block_lse"]), rtol=0, atol=1e-12)
    d = O.dense_causal_fwd(q, k, v, cu, sink=sink, scale=sc)
    np.testing.assert_allclose(d["lse"], e["dense_sink_lse"], atol=1e-12)
    np.testing.assert_allclose(d["out"], e["dense_sink_out"], atol=1e-12)
    d0 = O.dense_causal_fwd(q, k, v, cu, sink=None, scale=sc)
    np.testing.assert_allclose(d0["lse"], e["dense_nosink_lse"], atol=1e-12)
    np.testing.assert_allclose(d0["out"], e["dense_nosink_out"], atol=1e-12)
    s = O.sparse_mqa_fwd(q, k, v, np.array(e["sparse_idx"]), cu, B, sink=sink, scale=sc)
    np.testing.assert_allclose(s["lse"], e["sparse_lse"], atol=1e-12)
    np.testing.assert_allclose(s["out"], e["sparse_out"], atol=1e-12)
    w = O.swa_mqa_fwd(q, k, v, cu, e["swa_window"], sink=sink, scale=sc)
    np.testing.assert_allclose(w["lse"], e["swa_lse"], atol=1e-12)
    np.testing.assert_allclose(w["out"], e["swa_out"], atol=1e-12)
    # K = 1 keeps only the own block: the same sparse_idx comes out of select
    idx = O.select_topk(bs["block_score"], cu, B, 1)
    np.testing.assert_array_equal(idx, e["sparse_idx"])


def test_golden_example_b_topk_tie_rule():
    ex = json.load(open(GOLD))["example_b"]
    q, k = np.array(ex["q"]), np.array(ex["k"])
    cu, B, K = ex["cu_seqlens"], ex["block_size"], ex["topk"]
    bs = O.block_score(q, k, cu, B, scale=ex["scale"])
    np.testing.assert_allclose(bs["block_score"][3], ex["expect"]["block_score_t3"], atol=1e-12)
    np.testing.assert_allclose(bs["block_score"][4], ex["expect"]["block_score_t4"], atol=1e-12)
    # blocks 1 and 2 of token 3 are an exact tie only in exact arithmetic;
    # feed the hand values so that the tie is exact in float64 too
    sc = bs["block_score"].copy()
    sc[3, :4] = [1 / 8, 2 / 8, 2 / 8, 3 / 8]
    idx = O.select_topk(sc, cu, B, K)
    np.testing.assert_array_equal(idx, ex["expect"]["idx"])


def test_golden_example_c_packed_docs():
    ex = json.load(open(GOLD))["example_c"]
    q, k, v = (np.array(ex[n]) for n in ("q", "k", "v"))
    cu, B = ex["cu_seqlens"], ex["block_size"]
    bs = O.block_score(q, k, cu, B, scale=ex["scale"])
    np.testing.assert_allclose(bs["lse"], ex["expect"]["lse"], atol=1e-12)
    np.testing.assert_allclose(bs["block_score"], ex["expect"]["block_score"], atol=1e-12)
    d = O.dense_causal_fwd(q, k, v, cu, sink=None, scale=ex["scale"])
    np.testing.assert_allclose(d["out"], ex["expect"]["dense_out"], atol=1e-12)


def test_window_one_closed_form():
    """W = 1: each query sees only itself; out = v_t * sigmoid(s_tt - sink)."""
    q, k, v, sink, cu = _inputs(40, 3, 8, 5, docs=[17, 23], seed=3)
    sink = np.array([-1.0, 0.5, 2.0])
    sc = 8 ** -0.5
    w = O.swa_mqa_fwd(q, k, v, cu, 1, sink=sink, scale=sc)
    s_tt = sc * np.einsum("thd,td->th", q, k)
    lse = np.logaddexp(s_tt, sink[None, :])
    np.testing.assert_allclose(w["lse"], lse, rtol=1e-13)
    np.testing.assert_allclose(w["out"], (np.exp(s_tt - lse))[:, :, None] * v[:, None, :],
                               rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# library special cases
# ---------------------------------------------------------------------------

def _masked_logits(q, k, cu, sc):
    T = q.shape[0]
    s = sc * np.einsum("thd,jd->thj", q, k)
    mask = np.zeros((T, T), dtype=bool)
    for bos, eos in O.doc_bounds(cu):
        for t in range(bos, eos):
            mask[t, bos:t + 1] = True
    return np.where(mask[:, None, :], s, -np.inf), mask


def test_lse_matches_torch_logsumexp():
    q, k, v, sink, cu = _inputs(70, 3, 16, 8, docs=[29, 41], seed=1)
    sc = 16 ** -0.5
    bs = O.block_score(q, k, cu, 8, scale=sc)
    logits, _ = _masked_logits(q, k, cu, sc)
    ref = torch.logsumexp(torch.from_numpy(logits), dim=-1).numpy()
    np.testing.assert_allclose(bs["lse"], ref, rtol=1e-14, atol=1e-14)
    # per-block LSE against logsumexp over each block's slice of the logits
    for t in (0, 28, 29, 45, 69):
        bos = 0 if t < 29 else 29
        for b in range((t - bos) // 8 + 1):
            lo, hi = bos + 8 * b, min(bos + 8 * (b + 1), t + 1)
            ref_b = torch.logsumexp(torch.from_numpy(logits[t, :, lo:hi]), dim=-1).numpy()
            np.testing.assert_allclose(bs["block_lse"][t, :, b], ref_b, rtol=1e-14)


def _sdpa(q, k, v, mask, sc):
    """torch float64 SDPA with a boolean [T, T] mask, MQA via broadcast."""
    Q = torch.from_numpy(q).permute(1, 0, 2)              # [H, T, Dk]
    K = torch.from_numpy(k)[None].expand(q.shape[1], -1, -1)
    V = torch.from_numpy(v)[None].expand(q.shape[1], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(
        Q, K, V, attn_mask=torch.from_numpy(mask), scale=sc)
    return o.permute(1, 0, 2).numpy()


def test_no_sink_dense_matches_torch_sdpa_causal():
    q, k, v, _, cu = _inputs(64, 4, 16, 12, seed=2)
    sc = 16 ** -0.5
    d = O.dense_causal_fwd(q, k, v, cu, sink=None, scale=sc)
    Q = torch.from_numpy(q).permute(1, 0, 2)
    K = torch.from_numpy(k)[None].expand(4, -1, -1)
    V = torch.from_numpy(v)[None].expand(4, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=sc)
    np.testing.assert_allclose(d["out"], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)
    # sink = -inf is the same as no sink
    dn = O.dense_causal_fwd(q, k, v, cu, sink=np.full(4, -np.inf), scale=sc)
    np.testing.assert_array_equal(dn["out"], d["out"])
    np.testing.assert_array_equal(dn["lse"], d["lse"])


def test_no_sink_sparse_and_swa_match_torch_sdpa_masked():
    T, B, K = 72, 8, 3
    q, k, v, _, cu = _inputs(T, 3, 16, 8, docs=[30, 42], seed=4)
    sc = 0.3
    bs = O.block_score(q, k, cu, B, scale=sc)
    idx = O.select_topk(bs["block_score"], cu, B, K)
    s = O.sparse_mqa_fwd(q, k, v, idx, cu, B, sink=None, scale=sc)
    mask = np.array(loops.mask_from_blocks(T, cu, idx, B))
    np.testing.assert_allclose(s["out"], _sdpa(q, k, v, mask, sc), rtol=1e-12, atol=1e-13)
    w = O.swa_mqa_fwd(q, k, v, cu, 9, sink=None, scale=sc)
    maskw = np.array(loops.mask_from_window(T, cu, 9))
    np.testing.assert_allclose(w["out"], _sdpa(q, k, v, maskw, sc), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

def test_block_mass_sums_to_heads():
    """Per head the block masses sum to 1, so the scores sum to H (no sink
    in step 1)."""
    q, k, v, sink, cu = _inputs(90, 5, 8, 4, docs=[7, 33, 50], seed=5)
    bs = O.block_score(q, k, cu, 16, scale=0.5)
    np.testing.assert_allclose(bs["block_score"].sum(axis=1), 5.0, rtol=1e-12)
    per_head = np.exp(bs["block_lse"] - bs["lse"][:, :, None]).sum(axis=2)
    np.testing.assert_allclose(per_head, 1.0, rtol=1e-12)
    # future blocks carry nothing
    for bos, eos in O.doc_bounds(cu):
        for t in range(bos, eos):
            bq = (t - bos) // 16
            assert np.all(bs["block_score"][t, bq + 1:] == 0.0)
            assert np.all(np.isneginf(bs["block_lse"][t, :, bq + 1:]))


@pytest.mark.parametrize("docs", [[100], [37, 63], [5, 64, 31]])
def test_full_coverage_sparse_equals_dense_bitwise(docs):
    T = sum(docs)
    q, k, v, sink, cu = _inputs(T, 4, 16, 8, docs=docs, seed=6)
    B = 16
    nbmax = max((n + B - 1) // B for n in docs)
    bs = O.block_score(q, k, cu, B)
    idx = O.select_topk(bs["block_score"], cu, B, nbmax)
    s = O.sparse_mqa_fwd(q, k, v, idx, cu, B, sink=sink)
    d = O.dense_causal_fwd(q, k, v, cu, sink=sink)
    assert np.array_equal(s["out"], d["out"]) and np.array_equal(s["lse"], d["lse"])


@pytest.mark.parametrize("docs", [[100], [37, 63]])
def test_wide_window_equals_dense_bitwise(docs):
    T = sum(docs)
    q, k, v, sink, cu = _inputs(T, 4, 16, 8, docs=docs, seed=7)
    w = O.swa_mqa_fwd(q, k, v, cu, max(docs), sink=sink)
    d = O.dense_causal_fwd(q, k, v, cu, sink=sink)
    assert np.array_equal(w["out"], d["out"]) and np.array_equal(w["lse"], d["lse"])


@pytest.mark.parametrize("sink_val", [-3.0, 0.0, 8.0])
def test_sink_closed_form(sink_val):
    """lse_sink = logaddexp(lse_plain, sink); out_sink = out_plain *
    (1 - exp(sink - lse_sink)): the sink only adds to the denominator."""
    q, k, v, _, cu = _inputs(48, 3, 16, 8, docs=[20, 28], seed=8)
    sink = np.array([sink_val, sink_val - 1.0, sink_val + 0.5])
    B, K = 8, 2
    bs = O.block_score(q, k, cu, B)
    idx = O.select_topk(bs["block_score"], cu, B, K)
    for fn in (lambda s: O.sparse_mqa_fwd(q, k, v, idx, cu, B, sink=s),
               lambda s: O.swa_mqa_fwd(q, k, v, cu, 6, sink=s)):
        p, w = fn(None), fn(sink)
        lse = np.logaddexp(p["lse"], sink[None, :])
        np.testing.assert_allclose(w["lse"], lse, rtol=1e-13)
        np.testing.assert_allclose(w["lse_nosink"], p["lse"], rtol=1e-13)
        scale = 1.0 - np.exp(sink[None, :] - lse)
        np.testing.assert_allclose(w["out"], p["out"] * scale[:, :, None], rtol=1e-11, atol=1e-14)


def test_doc_isolation():
    """Packed outputs equal per-document outputs; perturbing one document's
    k and v leaves every other document's outputs bitwise unchanged."""
    docs = [19, 33, 12]
    T = sum(docs)
    q, k, v, sink, cu = _inputs(T, 3, 16, 8, docs=docs, seed=9)
    B, K, W = 8, 3, 10
    bs = O.block_score(q, k, cu, B)
    idx = O.select_topk(bs["block_score"], cu, B, K)
    sp = O.sparse_mqa_fwd(q, k, v, idx, cu, B, sink=sink)
    sw = O.swa_mqa_fwd(q, k, v, cu, W, sink=sink)
    for bos, eos in O.doc_bounds(cu):
        one = [0, eos - bos]
        bs1 = O.block_score(q[bos:eos], k[bos:eos], one, B)
        nb = bs1["block_score"].shape[1]
        np.testing.assert_array_equal(bs1["block_score"], bs["block_score"][bos:eos, :nb])
        idx1 = O.select_topk(bs1["block_score"], one, B, K)
        np.testing.assert_array_equal(idx1, idx[bos:eos])
        sp1 = O.sparse_mqa_fwd(q[bos:eos], k[bos:eos], v[bos:eos], idx1, one, B, sink=sink)
        np.testing.assert_array_equal(sp1["out"], sp["out"][bos:eos])
        sw1 = O.swa_mqa_fwd(q[bos:eos], k[bos:eos], v[bos:eos], one, W, sink=sink)
        np.testing.assert_array_equal(sw1["out"], sw["out"][bos:eos])
    k2, v2 = k.copy(), v.copy()
    k2[19:52] += 1.0
    v2[19:52] -= 2.0
    bs2 = O.block_score(q, k2, cu, B)
    sp2 = O.sparse_mqa_fwd(q, k2, v2, idx, cu, B, sink=sink)
    sw2 = O.swa_mqa_fwd(q, k2, v2, cu, W, sink=sink)
    for a, b in ((bs2["block_score"], bs["block_score"]), (sp2["out"], sp["out"]),
                 (sw2["out"], sw["out"])):
        np.testing.assert_array_equal(a[:19], b[:19])
        np.testing.assert_array_equal(a[52:], b[52:])
        assert not np.array_equal(a[19:52], b[19:52])


def test_topk_bruteforce_with_ties():
    """Sort-based selection equals exhaustive search (max summed score,
    lexicographically smallest on ties) on integer scores full of ties."""
    rng = np.random.default_rng(10)
    docs = [23, 41]
    cu = [0, 23, 64]
    B = 4
    for K in (2, 3, 4, 6, 11):
        scores = rng.integers(0, 4, size=(64, 11)).astype(np.float64)
        idx = O.select_topk(scores, cu, B, K)
        for t in range(64):
            bos = 0 if t < 23 else 23
            bq = (t - bos) // B
            ref = loops.topk_bruteforce(list(scores[t]), bq, K)
            got = [int(x) for x in idx[t] if x >= 0]
            assert got == ref, (K, t, got, ref)
            assert list(idx[t][len(got):]) == [-1] * (K - len(got))


def test_topk_monotonic():
    """Raising a selected block's score keeps it selected; raising a
    rejected block far enough brings it in."""
    rng = np.random.default_rng(11)
    cu = [0, 64]
    scores = rng.random((64, 16))
    idx = O.select_topk(scores, cu, 4, 5)
    t = 63
    for b in idx[t]:
        s2 = scores.copy()
        s2[t, b] += 0.5
        assert b in O.select_topk(s2, cu, 4, 5)[t]
    rejected = [b for b in range(16) if b not in idx[t]]
    s3 = scores.copy()
    s3[t, rejected[0]] = 10.0
    assert rejected[0] in O.select_topk(s3, cu, 4, 5)[t]


def test_block_scores_match_loops():
    docs = [13, 27]
    q, k, v, sink, cu = _inputs(40, 2, 6, 3, docs=docs, seed=12)
    sc = 0.7
    bs = O.block_score(q, k, cu, 4, scale=sc)
    lse, blse, score = loops.block_scores(q.tolist(), k.tolist(), cu, 4, sc)
    np.testing.assert_allclose(bs["lse"], lse, rtol=1e-13)
    np.testing.assert_allclose(bs["block_score"], score, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(bs["block_lse"], blse, rtol=1e-13)


@pytest.mark.parametrize("with_sink", [False, True])
def test_attention_matches_loops(with_sink):
    docs = [21, 9, 30]
    T = sum(docs)
    q, k, v, sink, cu = _inputs(T, 2, 6, 5, docs=docs, seed=13)
    sink = sink if with_sink else None
    sc = 0.4
    B, K, W = 4, 3, 5
    bs = O.block_score(q, k, cu, B, scale=sc)
    idx = O.select_topk(bs["block_score"], cu, B, K)
    s = O.sparse_mqa_fwd(q, k, v, idx, cu, B, sink=sink, scale=sc)
    mask = loops.mask_from_blocks(T, cu, idx, B)
    out, lse = loops.masked_attention(q.tolist(), k.tolist(), v.tolist(), mask,
                                      None if sink is None else sink.tolist(), sc)
    np.testing.assert_allclose(s["out"], out, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(s["lse"], lse, rtol=1e-13)
    w = O.swa_mqa_fwd(q, k, v, cu, W, sink=sink, scale=sc)
    mask = loops.mask_from_window(T, cu, W)
    out, lse = loops.masked_attention(q.tolist(), k.tolist(), v.tolist(), mask,
                                      None if sink is None else sink.tolist(), sc)
    np.testing.assert_allclose(w["out"], out, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(w["lse"], lse, rtol=1e-13)


@pytest.mark.parametrize("K", [1, 2, 5, 8])
def test_selection_follows_a_planted_block_order(K):
    """Scores with a planted order (synth.plant_block_order: every logit of a
    key in block b gains 3 * perm[b] natural-log units) must make the
    oracle's step 1 + step 2 pick exactly the blocks that the selection rule
    ("HySparse MQA sparse attention ..." pull request, hs_select_topk: own
    block and block 0 forced, the rest by descending block score, ties to
    the lower id) implies for that order, computed here without any scores.
    A reversed sort, a dropped forced block or a wrong causal limit fails."""
    base = synth.make_inputs(300, 4, 64, 48, dtype=torch.float32, seed=21,
                             doc_lengths=[0, 170, 0, 130])
    inp, perms = synth.plant_block_order(base, 16, gap=3.0, seed=21)
    f = lambda t: t.double().numpy()
    cu = inp.cu_seqlens.tolist()
    bs = O.block_score(f(inp.q), f(inp.k), cu, 16)
    idx = O.select_topk(bs["block_score"], cu, 16, K, total_tokens=300)
    np.testing.assert_array_equal(idx, P.planted_selection(cu, perms, 16, K))


def test_selection_structure():
    """Edge cases of the selection rule: forced blocks present, sizes right,
    docs shorter than a block, k larger than the candidate count."""
    docs = [3, 16, 17, 70]
    T = sum(docs)
    q, k, v, sink, cu = _inputs(T, 2, 8, 4, docs=docs, seed=14)
    B = 16
    bs = O.block_score(q, k, cu, B)
    for K in (1, 2, 3, 5, 8):
        idx = O.select_topk(bs["block_score"], cu, B, K)
        for bos, eos in O.doc_bounds(cu):
            for t in range(bos, eos):
                bq = (t - bos) // B
                sel = [int(x) for x in idx[t] if x >= 0]
                assert sel == sorted(set(sel))
                assert bq in sel
                if K >= 2:
                    assert 0 in sel
                assert len(sel) == min(K, bq + 1)
                assert all(0 <= b <= bq for b in sel)


def test_sampled_rows_match_full():
    q, k, v, sink, cu = _inputs(50, 2, 8, 4, docs=[20, 30], seed=15)
    rows = np.array([0, 7, 19, 20, 49])
    full = O.block_score(q, k, cu, 8)
    part = O.block_score(q, k, cu, 8, rows=rows)
    np.testing.assert_array_equal(part["block_score"], full["block_score"][rows])
    idx = O.select_topk(full["block_score"], cu, 8, 3)
    idx_p = O.select_topk(part["block_score"], cu, 8, 3, rows=rows, total_tokens=50)
    np.testing.assert_array_equal(idx_p, idx[rows])
    s = O.sparse_mqa_fwd(q, k, v, idx, cu, 8, sink=sink)
    sp = O.sparse_mqa_fwd(q, k, v, idx[rows], cu, 8, sink=sink, rows=rows)
    np.testing.assert_array_equal(sp["out"], s["out"][rows])


# ---------------------------------------------------------------------------
# the full layer's forward with block scores
# ---------------------------------------------------------------------------

def test_full_layer_matches_torch_sdpa_and_logsumexp():
    """out against torch float64 causal SDPA document by document; lse and
    every block's LSE against torch.logsumexp over the masked logits."""
    docs = [29, 41]
    q, k, v, _, cu = _inputs(70, 3, 16, 8, docs=docs, seed=31)
    sc = 0.35
    f = O.full_layer_fwd(q, k, v, cu, 8, scale=sc)
    for bos, eos in O.doc_bounds(cu):
        Q = torch.from_numpy(q[bos:eos]).permute(1, 0, 2)
        K = torch.from_numpy(k[bos:eos])[None].expand(3, -1, -1)
        V = torch.from_numpy(v[bos:eos])[None].expand(3, -1, -1)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=sc)
        np.testing.assert_allclose(f["out"][bos:eos], ref.permute(1, 0, 2).numpy(), rtol=1e-12,
                                   atol=1e-13)
    logits, _ = _masked_logits(q, k, cu, sc)
    ref = torch.logsumexp(torch.from_numpy(logits), dim=-1).numpy()
    np.testing.assert_allclose(f["lse"], ref, rtol=1e-14, atol=1e-14)
    for t in (0, 7, 8, 28, 29, 37, 69):
        bos = 0 if t < 29 else 29
        for b in range((t - bos) // 8 + 1):
            lo, hi = bos + 8 * b, min(bos + 8 * (b + 1), t + 1)
            ref_b = torch.logsumexp(torch.from_numpy(logits[t, :, lo:hi]), dim=-1).numpy()
            np.testing.assert_allclose(f["block_lse"][t, :, b], ref_b, rtol=1e-14)


def test_full_layer_block_closed_forms():
    """Per head the block LSEs log-sum-exp to the row LSE, so the scores sum
    to H; blocks past the query's own carry -inf / 0."""
    q, k, v, _, cu = _inputs(90, 5, 8, 4, docs=[7, 33, 50], seed=32)
    f = O.full_layer_fwd(q, k, v, cu, 16, scale=0.5)
    lse_b = torch.logsumexp(torch.from_numpy(f["block_lse"]), dim=-1).numpy()
    np.testing.assert_allclose(lse_b, f["lse"], rtol=1e-13)
    np.testing.assert_allclose(f["block_score"].sum(axis=1), 5.0, rtol=1e-12)
    for bos, eos in O.doc_bounds(cu):
        for t in range(bos, eos):
            bq = (t - bos) // 16
            assert np.all(f["block_score"][t, bq + 1:] == 0.0)
            assert np.all(np.isneginf(f["block_lse"][t, :, bq + 1:]))


def test_full_layer_matches_loops():
    """Brute force: the pure-loop block scorer and the loop attention over
    an explicit causal mask."""
    docs = [13, 27]
    T = sum(docs)
    q, k, v, _, cu = _inputs(T, 2, 6, 3, docs=docs, seed=33)
    sc = 0.7
    f = O.full_layer_fwd(q, k, v, cu, 4, scale=sc)
    lse, blse, score = loops.block_scores(q.tolist(), k.tolist(), cu, 4, sc)
    np.testing.assert_allclose(f["lse"], lse, rtol=1e-13)
    np.testing.assert_allclose(f["block_score"], score, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(f["block_lse"], blse, rtol=1e-13)
    out, lse2 = loops.masked_attention(q.tolist(), k.tolist(), v.tolist(),
                                       loops.mask_causal(T, cu), None, sc)
    np.testing.assert_allclose(f["out"], out, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(f["lse"], lse2, rtol=1e-13)


def test_full_layer_rows_and_separate_steps():
    """Sampled rows equal the full result; the fused definition equals step
    1 plus dense causal attention without a sink computed separately."""
    docs = [50, 14, 36]
    q, k, v, _, cu = _inputs(100, 4, 16, 12, docs=docs, seed=34)
    f = O.full_layer_fwd(q, k, v, cu, 16)
    rows = np.array([0, 13, 49, 50, 63, 64, 99])
    fr = O.full_layer_fwd(q, k, v, cu, 16, rows=rows)
    for key in ("out", "lse", "block_lse", "block_score"):
        np.testing.assert_array_equal(fr[key], f[key][rows])
    bs = O.block_score(q, k, cu, 16)
    d = O.dense_causal_fwd(q, k, v, cu, sink=None)
    np.testing.assert_allclose(f["block_score"], bs["block_score"], rtol=1e-13, atol=1e-16)
    np.testing.assert_array_equal(np.isneginf(f["block_lse"]), np.isneginf(bs["block_lse"]))
    np.testing.assert_allclose(f["out"], d["out"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(f["lse"], d["lse"], rtol=1e-14)


# ---------------------------------------------------------------------------
# the SWA layer: window branch + sparse branch on the shared KV, gated sum
# ---------------------------------------------------------------------------

def _layer_inputs(T, H, dk, dv, docs, seed):
    q, k, v, sink, cu = _inputs(T, H, dk, dv, docs=docs, seed=seed)
    _, ks, vs, sink2, _ = _inputs(T, H, dk, dv, docs=docs, seed=seed + 100)
    g = np.random.default_rng(seed).uniform(0.0, 1.0, size=(2, T, H))
    return q, k, v, ks, vs, sink, sink2, g[0], g[1], cu


def test_swa_layer_matches_torch_sdpa_gated_sum():
    """No sinks: each branch is torch float64 SDPA over its own boolean mask
    and its own KV; the layer output is the gated sum."""
    T, B, K, W = 72, 8, 3, 9
    docs = [30, 42]
    q, k, v, ks, vs, _, _, gw, gs, cu = _layer_inputs(T, 3, 16, 8, docs, 41)
    sc = 0.3
    # block lists chosen on other queries (the full layer's), here a fixed seed
    qf = _inputs(T, 3, 16, 8, docs=docs, seed=99)[0]
    idx = O.select_topk(O.block_score(qf, ks, cu, B, scale=sc)["block_score"], cu, B, K)
    f = O.swa_layer_fwd(q, k, v, ks, vs, idx, cu, W, B, gate_swa=gw, gate_sparse=gs, scale=sc)
    mw = np.array(loops.mask_from_window(T, cu, W))
    mb = np.array(loops.mask_from_blocks(T, cu, idx, B))
    ref = gw[:, :, None] * _sdpa(q, k, v, mw, sc) + gs[:, :, None] * _sdpa(q, ks, vs, mb, sc)
    np.testing.assert_allclose(f["out"], ref, rtol=1e-12, atol=1e-13)


def test_swa_layer_gates_select_branches():
    """Gates (1, 0) give the window branch on the layer's own KV, (0, 1) the
    sparse branch on the shared KV, missing gates their plain sum; the lse
    of each branch carries its own sink."""
    T, B, K, W = 100, 16, 3, 20
    docs = [50, 14, 36]
    q, k, v, ks, vs, s1, s2, _, _, cu = _layer_inputs(T, 4, 16, 12, docs, 42)
    idx = O.select_topk(O.block_score(q, ks, cu, B)["block_score"], cu, B, K)
    one, zero = np.ones((T, 4)), np.zeros((T, 4))
    w = O.swa_mqa_fwd(q, k, v, cu, W, sink=s1)
    sp = O.sparse_mqa_fwd(q, ks, vs, idx, cu, B, sink=s2)
    a = O.swa_layer_fwd(q, k, v, ks, vs, idx, cu, W, B, s1, s2, gate_swa=one, gate_sparse=zero)
    b = O.swa_layer_fwd(q, k, v, ks, vs, idx, cu, W, B, s1, s2, gate_swa=zero, gate_sparse=one)
    c = O.swa_layer_fwd(q, k, v, ks, vs, idx, cu, W, B, s1, s2)
    np.testing.assert_array_equal(a["out"], w["out"])
    np.testing.assert_array_equal(b["out"], sp["out"])
    np.testing.assert_array_equal(c["out"], w["out"] + sp["out"])
    np.testing.assert_array_equal(c["lse_swa"], w["lse"])
    np.testing.assert_array_equal(c["lse_sparse"], sp["lse"])
    # the shared KV reaches the output only through the sparse branch
    ks2 = ks + 1.0
    d = O.swa_layer_fwd(q, k, v, ks2, vs, idx, cu, W, B, s1, s2, gate_swa=one, gate_sparse=zero)
    np.testing.assert_array_equal(d["out"], a["out"])
    e = O.swa_layer_fwd(q, k, v, ks2, vs, idx, cu, W, B, s1, s2)
    assert np.abs(e["out"] - c["out"]).max() > 1e-3


def test_swa_layer_matches_loops_and_rows():
    docs = [21, 9, 30]
    T = sum(docs)
    q, k, v, ks, vs, s1, s2, gw, gs, cu = _layer_inputs(T, 2, 6, 5, docs, 43)
    sc, B, K, W = 0.4, 4, 3, 5
    idx = O.select_topk(O.block_score(q, ks, cu, B, scale=sc)["block_score"], cu, B, K)
    f = O.swa_layer_fwd(q, k, v, ks, vs, idx, cu, W, B, s1, s2, gw, gs, scale=sc)
    ow, lw = loops.masked_attention(q.tolist(), k.tolist(), v.tolist(),
                                    loops.mask_from_window(T, cu, W), s1.tolist(), sc)
    osp, lsp = loops.masked_attention(q.tolist(), ks.tolist(), vs.tolist(),
                                      loops.mask_from_blocks(T, cu, idx, B), s2.tolist(), sc)
    ref = gw[:, :, None] * np.array(ow) + gs[:, :, None] * np.array(osp)
    np.testing.assert_allclose(f["out"], ref, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(f["lse_swa"], lw, rtol=1e-13)
    np.testing.assert_allclose(f["lse_sparse"], lsp, rtol=1e-13)
    rows = np.array([0, 5, 20, 21, 29, 30, 59])
    fr = O.swa_layer_fwd(q, k, v, ks, vs, idx[rows], cu, W, B, s1, s2, gw, gs, scale=sc, rows=rows)
    for key in ("out", "lse_swa", "lse_sparse"):
        np.testing.assert_array_equal(fr[key], f[key][rows])
