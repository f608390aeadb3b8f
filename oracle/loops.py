"""Pure-Python loop restatements of the HySparse forward steps, for brute
force on tiny inputs (T <= 64, few heads, small head dims).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).  These functions are
written independently of ``oracle.hysparse`` -- different structure, no
NumPy, Python ``math`` only -- so that agreement between the two pins both.

* attention is computed from an explicit [T, T] boolean mask (built from
  the selected blocks or from the window), one (query, head) pair at a
  time;
* top-k is found by enumerating every subset of the free candidates.

Sources are the same pages as ``oracle.hysparse`` ("HySparse MQA sparse
attention ...", PaddleFleet pull request 1470, "Core" list and per-file
table; "Support attn sink in fa3", pull request 1415, for the sink as a
softmax offset).
"""

from __future__ import annotations

import itertools
import math


def _dot(a, b):
    acc = 0.0
    for x, y in zip(a, b):
        acc += float(x) * float(y)
    return acc


def docs_of(cu):
    cu = [int(x) for x in cu]
    return [(cu[i], cu[i + 1]) for i in range(len(cu) - 1)]


def doc_index(cu, t):
    for d, (b, e) in enumerate(docs_of(cu)):
        if b <= t < e:
            return d
    raise IndexError(t)


def mask_from_blocks(T, cu, idx, block_size):
    """mask[t][j] is True when query t attends key j: j is in a selected
    block of t's document and j <= t."""
    mask = [[False] * T for _ in range(T)]
    for t in range(T):
        bos, eos = docs_of(cu)[doc_index(cu, t)]
        for b in idx[t]:
            b = int(b)
            if b < 0:
                continue
            for j in range(bos + b * block_size, bos + (b + 1) * block_size):
                if bos <= j < eos and j <= t:
                    mask[t][j] = True
    return mask


def mask_from_window(T, cu, window):
    mask = [[False] * T for _ in range(T)]
    for t in range(T):
        bos, _ = docs_of(cu)[doc_index(cu, t)]
        for j in range(T):
            if bos <= j <= t and t - j < window:
                mask[t][j] = True
    return mask


def mask_causal(T, cu):
    mask = [[False] * T for _ in range(T)]
    for t in range(T):
        bos, _ = docs_of(cu)[doc_index(cu, t)]
        for j in range(bos, t + 1):
            mask[t][j] = True
    return mask


def masked_attention(q, k, v, mask, sink, scale):
    """out[t][h][:], lse[t][h] from a dense mask, one softmax per (t, h).

    q: nested lists [T][H][Dk]; k: [T][Dk]; v: [T][Dv]; sink: [H] or None.
    """
    T = len(q)
    H = len(q[0])
    Dv = len(v[0])
    out = [[[0.0] * Dv for _ in range(H)] for _ in range(T)]
    lse = [[0.0] * H for _ in range(T)]
    for t in range(T):
        for h in range(H):
            logits = []
            for j in range(T):
                if mask[t][j]:
                    logits.append((j, scale * _dot(q[t][h], k[j])))
            sk = -math.inf if sink is None else float(sink[h])
            top = max([s for _, s in logits] + [sk])
            denom = sum(math.exp(s - top) for _, s in logits)
            if sk != -math.inf:
                denom += math.exp(sk - top)
            l = top + math.log(denom)
            lse[t][h] = l
            for j, s in logits:
                w = math.exp(s - l)
                for c in range(Dv):
                    out[t][h][c] += w * float(v[j][c])
    return out, lse


def block_scores(q, k, cu, block_size, scale):
    """(lse[t][h], block_lse[t][h][b], score[t][b]) by direct summation of
    exp over the causal keys of every block; no sink."""
    T = len(q)
    H = len(q[0])
    nbmax = max((e - b + block_size - 1) // block_size for b, e in docs_of(cu))
    lse = [[0.0] * H for _ in range(T)]
    blse = [[[-math.inf] * nbmax for _ in range(H)] for _ in range(T)]
    score = [[0.0] * nbmax for _ in range(T)]
    for t in range(T):
        bos, eos = docs_of(cu)[doc_index(cu, t)]
        for h in range(H):
            tot = 0.0
            sums = [0.0] * nbmax
            for j in range(bos, t + 1):
                e = math.exp(scale * _dot(q[t][h], k[j]))
                tot += e
                sums[(j - bos) // block_size] += e
            lse[t][h] = math.log(tot)
            for b in range(nbmax):
                if sums[b] > 0.0:
                    blse[t][h][b] = math.log(sums[b])
                    score[t][b] += sums[b] / tot
    return lse, blse, score


def topk_bruteforce(scores_row, bq, k):
    """Best block set for one query by exhaustive search.

    Forced blocks {bq, 0} are in; among all subsets of the free candidates
    1..bq-1 of the right size, keep the one with the largest summed score;
    among equal sums keep the lexicographically smallest sorted id list
    (the lower-index tie rule).  Returns an ascending list.
    """
    if bq + 1 <= k:
        return list(range(bq + 1))
    forced = [0, bq] if bq > 0 else [0]
    if k < len(forced):
        return [bq]
    free = list(range(1, bq))
    need = k - len(forced)
    best = None
    for combo in itertools.combinations(free, need):
        total = sum(scores_row[b] for b in combo)
        key = (-total, sorted(combo))
        if best is None or key < best[0]:
            best = (key, combo)
    return sorted(forced + list(best[1]))
