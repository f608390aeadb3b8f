"""Plain float64 CPU definition of the HySparse MQA forward path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` call it.  It shares no code with the CUDA library.

Sources (web pages, cited by title and section):

* [HS]  "HySparse MQA sparse attention (FA4 block scoring + SWA MQA +
  block-sparse DSA gather)", PaddleFleet pull request 1470: the "Core" list
  (FA4-fused block scoring, SWA sliding-window MQA, block-sparse DSA gather
  with a learnable per-head attn_sink), the "FlashMLA sparse kernel
  constraints" section (absorbed-MLA MQA layout: one KV head, Dk = latent +
  RoPE, Dv = latent) and the Copilot per-file table (``pipeline.py``:
  top-k block selection after recovering the block score as
  ``exp(block_logit - lse)``; ``swa_attn.py``: default ``sm_scale``;
  ``windowed_mqa_attn*.py``: Dk != Dv and an optional attn_sink).
* [SINK] "Support attn sink in fa3", PaddleFleet pull request 1415, review
  thread on the dense path: the sink is a softmax offset, i.e. an extra
  logit that enters the softmax denominator and contributes no value row.
* [REV] Review comments on PaddleFleet pull request 1453 (the same code as
  1470): the block-score PyLayer takes a per-document ``block_bos`` tensor
  (blocks restart at every packed document) and saves ``out`` and ``lse``;
  the windowed kernel takes per-row ``bos``/``eos`` key ranges.
* [DISP] "Unified sparse attention API (dispatcher)" blog page, key points of
  the model-config section: a sparse pattern that covers every causal key is
  identical to dense causal attention.

Readings taken where the pages are silent:

* Block scoring carries no sink.  The block score of key block ``b`` for
  query ``t`` is the head-summed probability mass
  ``sum_h exp(blockLSE[t,h,b] - LSE[t,h])`` (natural log, scaled logits).
* Blocks are laid on each document separately, starting at its first token;
  the last block of a document may be partial.  Block ids are doc-local.
* Top-k always keeps the query's own block and the document's first block;
  they count toward k.  Remaining slots go to the highest scores, ties to
  the lower block id.  Output is ascending, padded with -1.
* The sink is a raw logit in the already-scaled space (not multiplied by the
  softmax scale); the returned ``lse`` includes it: ``lse = log(e^sink +
  sum_j e^{s_j})`` and ``out = sum_j e^{s_j - lse} v_j``.
* The sliding window of width W holds the W keys ending at the query:
  ``j`` in ``[max(bos, t - W + 1), t]``.

All arithmetic is float64.  Every function accepts an optional ``rows``
array of query-token indices and then returns results for those rows only,
in that order (used for sampled checks at large sizes).
"""

from __future__ import annotations

import math
from typing import Optional

import numpy as np

__all__ = [
    "RowSubset",
    "doc_bounds",
    "num_blocks",
    "block_score",
    "select_topk",
    "sparse_key_set",
    "window_key_set",
    "attend",
    "sparse_mqa_fwd",
    "swa_mqa_fwd",
    "dense_causal_fwd",
    "full_layer_fwd",
    "swa_layer_fwd",
]


# ---------------------------------------------------------------------------
# documents and blocks
# ---------------------------------------------------------------------------

def doc_bounds(cu_seqlens) -> list[tuple[int, int]]:
    """[(bos, eos), ...] for every packed document.

    ``cu_seqlens`` holds num_docs + 1 non-decreasing offsets starting at 0
    (the packed-sequence convention of [REV], ``packed_seq_params``).
    """
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    if not cu or cu[0] != 0:
        raise ValueError("cu_seqlens must start at 0")
    for a, b in zip(cu[:-1], cu[1:]):
        if b < a:
            raise ValueError("cu_seqlens must be non-decreasing")
    return list(zip(cu[:-1], cu[1:]))


def num_blocks(length: int, block_size: int) -> int:
    """Blocks of a document of ``length`` tokens (last one may be partial)."""
    return (length + block_size - 1) // block_size


def _doc_of_rows(cu_seqlens, total: int) -> np.ndarray:
    """Document index of every token."""
    doc = np.empty(total, dtype=np.int64)
    for d, (bos, eos) in enumerate(doc_bounds(cu_seqlens)):
        doc[bos:eos] = d
    return doc


def _rows(rows, total: int) -> np.ndarray:
    if rows is None:
        return np.arange(total, dtype=np.int64)
    return np.asarray(rows, dtype=np.int64).reshape(-1)


def _scale(scale: Optional[float], dk: int) -> float:
    """Softmax scale; a missing or non-positive value means Dk^-1/2, the
    default of the SWA wrapper in [HS] (per-file table, ``swa_attn.py``)."""
    if scale is None or scale <= 0:
        return 1.0 / math.sqrt(dk)
    return float(scale)


def _f64(x) -> np.ndarray:
    if isinstance(x, RowSubset):
        return x
    return np.asarray(x, dtype=np.float64)


class RowSubset:
    """q given only for some query tokens (sampled checks at sizes where a
    full float64 copy of q would not fit in host memory).  Indexing by a
    token returns its [H, Dk] float64 row; other tokens are absent."""

    def __init__(self, rows: dict, shape):
        self._rows = {int(t): np.asarray(v, dtype=np.float64) for t, v in rows.items()}
        self.shape = tuple(shape)

    def __getitem__(self, t):
        return self._rows[int(t)]


# ---------------------------------------------------------------------------
# step 1: block scoring
# ---------------------------------------------------------------------------

def block_score(q, k, cu_seqlens, block_size: int, scale=None, rows=None):
    """Causal block scoring ([HS] "Core": FA4-fused block scoring; per-file
    table, ``pipeline.py``: score = exp(block_logit - lse)).

    For query t of document d = [bos, eos), head h and doc-local block
    b <= bq(t) = (t - bos) // B::

        s_j            = scale * <q[t,h], k[j]>,            j in [bos, t]
        LSE[t,h]       = log sum_j exp(s_j)
        blockLSE[t,h,b]= log sum_{j in J_b(t)} exp(s_j)
        score[t,b]     = sum_h exp(blockLSE[t,h,b] - LSE[t,h])

    with J_b(t) = [bos + bB, min(bos + (b+1)B, eos)) intersected with
    [bos, t].  Blocks after bq(t) get blockLSE = -inf and score = 0, out to
    NBmax = max_d ceil(len_d / B).

    q: [T, H, Dk]; k: [T, Dk].  Returns a dict with ``lse`` [R, H],
    ``block_lse`` [R, H, NBmax] and ``block_score`` [R, NBmax] (float64).
    """
    q = _f64(q)
    k = _f64(k)
    T, H, Dk = q.shape
    B = int(block_size)
    sc = _scale(scale, Dk)
    bounds = doc_bounds(cu_seqlens)
    nbmax = max([num_blocks(e - b, B) for b, e in bounds] + [0])
    doc = _doc_of_rows(cu_seqlens, T)
    rr = _rows(rows, T)
    R = rr.shape[0]
    lse = np.empty((R, H))
    blse = np.full((R, H, nbmax), -np.inf)
    score = np.zeros((R, nbmax))
    for i, t in enumerate(rr):
        bos, eos = bounds[doc[t]]
        n = t - bos + 1                      # causal keys bos..t
        s = sc * (q[t] @ k[bos:t + 1].T)     # [H, n]
        m = s.max(axis=1)
        lse[i] = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
        nb = num_blocks(n, B)                # blocks 0..bq
        for b in range(nb):
            seg = s[:, b * B:min((b + 1) * B, n)]
            bm = seg.max(axis=1)
            blse[i, :, b] = bm + np.log(np.exp(seg - bm[:, None]).sum(axis=1))
        # head sum in increasing head order
        acc = np.zeros(nb)
        for h in range(H):
            acc = acc + np.exp(blse[i, h, :nb] - lse[i, h])
        score[i, :nb] = acc
    return {"lse": lse, "block_lse": blse, "block_score": score}


# ---------------------------------------------------------------------------
# step 2: top-k block selection
# ---------------------------------------------------------------------------

def select_topk(block_score_rows, cu_seqlens, block_size: int, topk: int,
                rows=None, total_tokens=None):
    """Per-query top-k key blocks inside the query's document ([HS]
    per-file table, ``pipeline.py``: top-k over the recovered block scores).

    Candidates are blocks 0..bq(t).  Forced blocks F = {bq, 0} (a single
    block when bq = 0) are always kept and count toward k.  If bq + 1 <= k
    every candidate is kept.  Otherwise the k - |F| best of the remaining
    candidates are added, ordered by (-score, block id), so that equal
    scores go to the lower id.  The result is ascending, padded with -1.

    ``block_score_rows`` holds one row per selected query (``rows`` order,
    all tokens when ``rows`` is None).  k >= 2 is required whenever some
    query has bq >= 1 (with k = 1 only the own block would fit, which the
    library rejects); here k = 1 keeps the own block only.
    """
    sc = _f64(block_score_rows)
    bounds = doc_bounds(cu_seqlens)
    T = bounds[-1][1] if bounds else 0
    if total_tokens is not None:
        T = int(total_tokens)
    doc = _doc_of_rows(cu_seqlens, T)
    rr = _rows(rows, T)
    B = int(block_size)
    K = int(topk)
    out = np.full((rr.shape[0], K), -1, dtype=np.int32)
    for i, t in enumerate(rr):
        bos, _ = bounds[doc[t]]
        bq = (t - bos) // B
        if bq + 1 <= K:
            chosen = list(range(bq + 1))
        else:
            forced = [bq] if bq == 0 else [0, bq]
            if K < len(forced):
                forced = [bq]
            others = [b for b in range(1, bq)]
            others.sort(key=lambda b: (-sc[i, b], b))
            chosen = sorted(forced + others[:K - len(forced)])
        out[i, :len(chosen)] = chosen
    return out


# ---------------------------------------------------------------------------
# key sets
# ---------------------------------------------------------------------------

def sparse_key_set(t: int, bos: int, eos: int, blocks, block_size: int):
    """Keys attended by query t given its selected doc-local blocks: the
    union of J_b(t) over blocks b >= 0, in ascending key order ([HS]
    per-file table, ``block_sparse_mqa_dsa.py``: block ids expanded to
    token indices)."""
    B = int(block_size)
    keys = []
    for b in sorted(int(x) for x in blocks if int(x) >= 0):
        lo = bos + b * B
        hi = min(bos + (b + 1) * B, eos, t + 1)
        keys.extend(range(lo, hi))
    return np.asarray(sorted(set(keys)), dtype=np.int64)


def window_key_set(t: int, bos: int, window: int):
    """Keys of the sliding window: the ``window`` keys ending at t, clipped
    at the document start ([REV]: windowed kernel rows carry bos/eos)."""
    lo = max(bos, t - int(window) + 1)
    return np.arange(lo, t + 1, dtype=np.int64)


# ---------------------------------------------------------------------------
# softmax attention with a sink
# ---------------------------------------------------------------------------

def attend(q_t, keys, k, v, sink, scale: float):
    """Softmax attention of one query token's H heads over ``keys``.

    s_j = scale * <q_t[h], k[j]>; the per-head sink logit enters the
    denominator only ([SINK]: softmax offset; [HS] "Core": learnable
    per-head attn_sink)::

        lse        = log(exp(sink_h) + sum_j exp(s_j))
        lse_nosink = log(sum_j exp(s_j))
        out[h]     = sum_j exp(s_j - lse) v[j]

    ``sink`` None means no sink (equivalently -inf).  An empty key set (an
    idx row without a usable block) gives out = 0 and lse = sink.  Returns
    (out [H, Dv], lse [H], lse_nosink [H]).
    """
    q_t = _f64(q_t)
    H = q_t.shape[0]
    kk = _f64(k)[keys]
    vv = _f64(v)[keys]
    sk = np.full(H, -np.inf) if sink is None else _f64(sink).reshape(H)
    if len(keys) == 0:  # no usable block: the softmax holds only the sink
        return np.zeros((H, vv.shape[1])), sk.copy(), np.full(H, -np.inf)
    s = scale * (q_t @ kk.T)                              # [H, n]
    m = np.maximum(s.max(axis=1), sk)                     # finite: n >= 1
    z = np.exp(s - m[:, None]).sum(axis=1)
    zs = np.exp(sk - m)
    lse = m + np.log(z + zs)
    lse_nosink = m + np.log(z)
    p = np.exp(s - lse[:, None])
    return p @ vv, lse, lse_nosink


def _attend_rows(q, k, v, cu_seqlens, sink, scale, rows, keyfn):
    q = _f64(q)
    T, H, Dk = q.shape
    Dv = np.asarray(v).shape[1]
    sc = _scale(scale, Dk)
    bounds = doc_bounds(cu_seqlens)
    doc = _doc_of_rows(cu_seqlens, T)
    rr = _rows(rows, T)
    out = np.empty((rr.shape[0], H, Dv))
    lse = np.empty((rr.shape[0], H))
    lse_ns = np.empty((rr.shape[0], H))
    kf = _f64(k)
    vf = _f64(v)
    for i, t in enumerate(rr):
        bos, eos = bounds[doc[t]]
        keys = keyfn(i, int(t), bos, eos)
        out[i], lse[i], lse_ns[i] = attend(q[t], keys, kf, vf, sink, sc)
    return {"out": out, "lse": lse, "lse_nosink": lse_ns}


def sparse_mqa_fwd(q, k, v, idx, cu_seqlens, block_size: int, sink=None,
                   scale=None, rows=None):
    """Block-sparse MQA forward ([HS] "Core": block-sparse DSA gather with
    a learnable per-head attn_sink).  ``idx`` [R, K] holds each query's
    doc-local block ids (-1 = unused slot), one row per query in ``rows``
    order.  Returns dict(out [R,H,Dv], lse [R,H], lse_nosink [R,H])."""
    idx = np.asarray(idx)

    def keys(i, t, bos, eos):
        return sparse_key_set(t, bos, eos, idx[i], block_size)

    return _attend_rows(q, k, v, cu_seqlens, sink, scale, rows, keys)


def swa_mqa_fwd(q, k, v, cu_seqlens, window: int, sink=None, scale=None,
                rows=None):
    """Sliding-window MQA forward ([HS] "Core": SWA sliding-window MQA;
    per-file table: Dk != Dv and an optional attn_sink)."""

    def keys(i, t, bos, eos):
        return window_key_set(t, bos, window)

    return _attend_rows(q, k, v, cu_seqlens, sink, scale, rows, keys)


def dense_causal_fwd(q, k, v, cu_seqlens, sink=None, scale=None, rows=None):
    """Dense causal MQA with sink inside each document: the reference point
    that full-coverage sparse and wide-window SWA must equal ([DISP])."""

    def keys(i, t, bos, eos):
        return np.arange(bos, t + 1, dtype=np.int64)

    return _attend_rows(q, k, v, cu_seqlens, sink, scale, rows, keys)


# ---------------------------------------------------------------------------
# the full layer's forward with its block scores (one pass over the logits)
# ---------------------------------------------------------------------------

def full_layer_fwd(q, k, v, cu_seqlens, block_size: int, scale=None, rows=None):
    """Forward of the full-attention layer that also scores the key blocks
    ([HS] "Core": FA4-fused block scoring, "HySparse full layer" bullet of
    the Copilot overview: the full layer produces the shared KV and the
    block indices; per-file table, ``block_score_fa4.py``: the block scorer
    is that layer's flash-attention forward emitting a scaled block_logit;
    [REV]: its PyLayer saves ``out`` and ``lse``).

    Per query t of document [bos, eos) and head h, over the causal keys
    j in [bos, t] with s_j = scale * <q[t,h], k[j]> and no sink::

        lse[t,h]          = log sum_j exp(s_j)
        out[t,h]          = sum_j exp(s_j - lse[t,h]) v[j]
        block_lse[t,h,b]  = log sum_{j in J_b(t)} exp(s_j)
        block_score[t,b]  = sum_h exp(block_lse[t,h,b] - lse[t,h])

    that is, dense causal attention and step 1's outputs from one set of
    logits.  Blocks after bq(t) get block_lse = -inf and score 0.  Returns
    dict(out [R,H,Dv], lse [R,H], block_lse [R,H,NBmax], block_score
    [R,NBmax]) in float64.
    """
    q = _f64(q)
    kf = _f64(k)
    vf = _f64(v)
    T, H, Dk = q.shape
    Dv = vf.shape[1]
    B = int(block_size)
    sc = _scale(scale, Dk)
    bounds = doc_bounds(cu_seqlens)
    nbmax = max([num_blocks(e - b, B) for b, e in bounds] + [0])
    doc = _doc_of_rows(cu_seqlens, T)
    rr = _rows(rows, T)
    R = rr.shape[0]
    out = np.empty((R, H, Dv))
    lse = np.empty((R, H))
    blse = np.full((R, H, nbmax), -np.inf)
    score = np.zeros((R, nbmax))
    for i, t in enumerate(rr):
        bos, eos = bounds[doc[t]]
        s = sc * (q[t] @ kf[bos:t + 1].T)                   # [H, n] causal logits
        m = s.max(axis=1)
        lse[i] = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
        out[i] = np.exp(s - lse[i][:, None]) @ vf[bos:t + 1]
        n = t - bos + 1
        nb = num_blocks(n, B)
        for b in range(nb):
            seg = s[:, b * B:min((b + 1) * B, n)]
            bm = seg.max(axis=1)
            blse[i, :, b] = bm + np.log(np.exp(seg - bm[:, None]).sum(axis=1))
        acc = np.zeros(nb)
        for h in range(H):                                 # increasing head order
            acc = acc + np.exp(blse[i, h, :nb] - lse[i, h])
        score[i, :nb] = acc
    return {"out": out, "lse": lse, "block_lse": blse, "block_score": score}


# ---------------------------------------------------------------------------
# the HySparse SWA layer: window branch + sparse branch on the shared KV
# ---------------------------------------------------------------------------

def swa_layer_fwd(q, k, v, k_shared, v_shared, idx, cu_seqlens, window: int,
                  block_size: int, sink_swa=None, sink_sparse=None, gate_swa=None,
                  gate_sparse=None, scale=None, rows=None):
    """Forward of the HySparse SWA layer ([HS] "What": NSA-style cooperating
    structures; Copilot overview: the SWA kernel is the SWA layer's main
    branch, the full layer produces the shared KV and the block indices;
    [REV] MQA test review: the SWA layer consumes shared_kv in a sparse
    branch).

    Reading taken (the pages name the two branches, not how they combine):
    as in NSA, each branch is its own softmax attention and the layer output
    is their gated sum::

        out[t,h] = gate_swa[t,h] * swa(q, k, v)[t,h]
                 + gate_sparse[t,h] * sparse(q, k_shared, v_shared, idx)[t,h]

    with the SWA layer's own queries q in both branches, each branch with its
    own optional per-head sink, and a missing gate meaning 1 (a plain sum).
    ``idx`` holds the block lists the full layer selected, one row per query
    in ``rows`` order (as ``sparse_mqa_fwd``); gates are [T, H].  Returns
    dict(out [R,H,Dv], lse_swa [R,H], lse_sparse [R,H]).
    """
    w = swa_mqa_fwd(q, k, v, cu_seqlens, window, sink=sink_swa, scale=scale, rows=rows)
    sp = sparse_mqa_fwd(q, k_shared, v_shared, idx, cu_seqlens, block_size, sink=sink_sparse,
                        scale=scale, rows=rows)
    T = np.asarray(k).shape[0]
    rr = _rows(rows, T)
    gw = np.ones((rr.shape[0], w["out"].shape[1])) if gate_swa is None else _f64(gate_swa)[rr]
    gs = np.ones_like(gw) if gate_sparse is None else _f64(gate_sparse)[rr]
    out = gw[:, :, None] * w["out"] + gs[:, :, None] * sp["out"]
    return {"out": out, "lse_swa": w["lse"], "lse_sparse": sp["lse"]}
