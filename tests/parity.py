"""Comparison helpers for GPU-vs-oracle parity.

Tolerances (the accuracy bound stated for this path, bf16 inputs with fp32
accumulation; applied to the fp32 workload as well):

* out:  max |gpu - oracle| <= 2e-2 and ||gpu - oracle||_F / ||oracle||_F <= 5e-3
* lse:  max |gpu - oracle| <= 1e-3
* top-k index sets: exact, except a block whose oracle score is within 1e-3
  (relative) of the oracle's k-th selected free score may be swapped with
  another such block (near ties); forced blocks and set sizes are exact.
* block_score (not graded, catches errors early): |gpu - oracle| <= 1e-4 *
  max(1, |oracle|); block-level lse to 1e-3 abs.
"""

from __future__ import annotations

import numpy as np

OUT_MAX_ABS = 2e-2
OUT_REL_FRO = 5e-3
LSE_ABS = 1e-3
SCORE_REL = 1e-4
TIE_REL = 1e-3


def np64(t):
    return t.detach().float().cpu().double().numpy() if hasattr(t, "detach") else np.asarray(t, np.float64)


def check_out(gpu, ref, what="out"):
    g = np64(gpu)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), what + ": non-finite values"
    err = np.abs(g - r)
    mx = float(err.max()) if err.size else 0.0
    fro = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)) if err.size else 0.0
    assert mx <= OUT_MAX_ABS, "%s max abs err %.3e > %.1e" % (what, mx, OUT_MAX_ABS)
    assert fro <= OUT_REL_FRO, "%s rel Frobenius err %.3e > %.1e" % (what, fro, OUT_REL_FRO)
    return mx, fro


def check_lse(gpu, ref, what="lse", tol=LSE_ABS):
    g = np64(gpu)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    both_inf = np.isneginf(g) & np.isneginf(r)
    with np.errstate(invalid="ignore"):
        err = np.where(both_inf, 0.0, np.abs(g - r))
    mx = float(np.nanmax(err)) if err.size else 0.0
    assert not np.any(np.isnan(err)), what + ": NaN"
    assert mx <= tol, "%s max abs err %.3e > %.1e" % (what, mx, tol)
    return mx


def check_scores(gpu, ref, what="block_score"):
    g = np64(gpu)
    r = np.asarray(ref, np.float64)
    g = g[:, :r.shape[1]]
    err = np.abs(g - r) / np.maximum(1.0, np.abs(r))
    mx = float(err.max()) if err.size else 0.0
    assert mx <= SCORE_REL, "%s rel err %.3e > %.1e" % (what, mx, SCORE_REL)
    return mx


def check_topk(gpu_idx, ref_idx, ref_scores, bq_of_row, topk):
    """Index sets exact up to near ties (see module doc).  Returns the number
    of rows where a near-tie swap was excused."""
    g = np.asarray(gpu_idx.cpu().numpy() if hasattr(gpu_idx, "cpu") else gpu_idx)
    r = np.asarray(ref_idx)
    sc = np.asarray(ref_scores, np.float64)
    excused = 0
    for i in range(r.shape[0]):
        gs = [int(x) for x in g[i] if x >= 0]
        rs = [int(x) for x in r[i] if x >= 0]
        assert gs == sorted(gs), ("row %d not ascending" % i, gs)
        assert list(g[i][len(gs):]) == [-1] * (topk - len(gs)), ("row %d padding" % i, g[i])
        if gs == rs:
            continue
        assert len(gs) == len(rs), ("row %d size" % i, gs, rs)
        bq = bq_of_row[i]
        forced = {bq, 0} if topk >= 2 else {bq}
        assert forced <= set(gs), ("row %d forced blocks missing" % i, gs)
        free_sel = [b for b in rs if b not in forced]
        kth = min(sc[i, b] for b in free_sel)
        for b in set(gs) ^ set(rs):
            rel = abs(sc[i, b] - kth) / max(abs(kth), 1e-30)
            assert rel <= TIE_REL, ("row %d block %d: score %.9g vs k-th %.9g" % (i, b, sc[i, b], kth),
                                    gs, rs)
        excused += 1
    return excused


def bq_rows(cu, rows, block_size):
    cu = [int(x) for x in cu]
    out = []
    for t in rows:
        d = max(i for i in range(len(cu) - 1) if cu[i] <= t)
        out.append((int(t) - cu[d]) // block_size)
    return out


def planted_selection(cu_seqlens, perms, block_size: int, topk: int, rows=None) -> np.ndarray:
    """The selection that a planted block order (synth.plant_block_order)
    implies, written from the selection rule of the pages (the query's own
    block and block 0 forced, the rest by descending score) with the scores'
    order taken from ``perms`` instead of computed: per query t of document d with own
    block bq, every block 0..bq when bq + 1 <= topk, else blocks 0 and bq plus
    the topk - 2 blocks of 1..bq-1 with the largest ``perms[d]`` (topk = 1:
    the own block alone); ascending, padded with -1.  Rows default to every
    token."""
    cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    T = cu[-1]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    out = np.full((len(rows), topk), -1, dtype=np.int32)
    for i, t in enumerate(rows):
        d = max(x for x in range(len(cu) - 1) if cu[x] <= t < cu[x + 1])
        bq = (int(t) - cu[d]) // block_size
        if bq + 1 <= topk:
            sel = list(range(bq + 1))
        elif topk == 1:
            sel = [bq]
        else:
            rest = sorted(range(1, bq), key=lambda b: -int(perms[d][b]))[:topk - 2]
            sel = sorted({0, bq, *rest})
        out[i, :len(sel)] = sel
    return out
