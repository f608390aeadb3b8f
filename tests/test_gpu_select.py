"""GPU parity of step 2 (hs_select_topk) on its own: score rows drawn here,
not by step 1, so that rows of every length class meet the kernel (the
register path for up to 32 x {1, 2, 4, 8, 16, 32} candidates and the
shared-memory path past 1024), with many exact ties.  Rows of more than 64
candidates with at most 32 free slots take the narrowed search (a pivot from
each lane's two largest keys, then a 64-entry list); the "ties" rows
overflow that list and take the full search, the "coarse" rows hold ties
around the pivot that often still fit in it.

Selection decides integers from fp32 scores, so both sides decide in fp32:
the oracle sorts the float64 images of the same fp32 values, which order
exactly as the fp32 values do (no -0.0 is drawn, the one value pair whose
fp32 keys would differ while their float64 images compare equal).  The
index output must be identical, element for element.
"""

import numpy as np
import pytest
import torch

import oracle.hysparse as O
from block_sparse_mqa_b200 import hs, synth

pytestmark = pytest.mark.gpu


def _scores(T, nb, kind, seed):
    """Seeded fp32 score rows, drawn on the GPU (the largest case holds 25 GB)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    u = torch.rand((T, nb), generator=g, device="cuda")
    if kind == "ties":      # small integers: almost every comparison is a tie
        return u.mul_(6.0).floor_()
    if kind == "flat":      # near-equal positive scores, as from N(0,1) inputs
        return u.mul_(2e-3).add_(1.0)
    if kind == "coarse":    # 48 levels: ties at the k-th value, short lists
        return u.mul_(48.0).floor_().add_(1.0)
    if kind == "mixed":     # exact zeros (underflow), tiny and large values
        z = torch.rand((T, nb), generator=g, device="cuda") < 0.2
        return u.mul_(105.0).sub_(100.0).exp_().masked_fill_(z, 0.0)
    raise ValueError(kind)


def _check(docs, B, K, kind, seed, rows=None):
    T = sum(docs)
    cu = synth.cu_from_lengths(docs)
    max_seqlen = max(docs)
    nb = hs.nbmax(max_seqlen, B)
    bs = _scores(T, nb + 3, kind, seed)  # nb_stride > NBmax: padding columns unread
    cu_dev = torch.as_tensor(cu, device="cuda", dtype=torch.int32)
    idx = hs.hs_select_topk(bs, cu_dev, max_seqlen, B, K)
    torch.cuda.synchronize()
    hs.poll_status()
    assert hs.last_path() == hs.HS_PATH_SIMT
    rr = np.arange(T) if rows is None else np.asarray(rows)
    rt = torch.as_tensor(rr, device="cuda")
    s64 = bs[rt].cpu().numpy().astype(np.float64)  # exact images of the fp32 scores
    ref = O.select_topk(s64, list(cu), B, K, rows=rr, total_tokens=T)
    np.testing.assert_array_equal(idx[rt].cpu().numpy(), ref)


@pytest.mark.parametrize("kind", ["ties", "coarse", "flat", "mixed"])
@pytest.mark.parametrize("B,K,docs", [
    (16, 4, [500, 0, 33]),          # up to 32 candidates: one register chunk
    (16, 2, [1000]),                 # k = 2: only the two forced blocks
    (16, 1, [300]),                  # k = 1: the own block alone
    (32, 9, [2048, 700]),            # 64 candidates: two chunks
    (64, 16, [8192, 64, 1]),         # 128: four chunks
    (16, 37, [4096, 5]),             # 256: eight chunks
    (64, 100, [32768]),              # 512: sixteen chunks
    (16, 256, [16384]),              # 1024: thirty-two chunks, topk at its maximum
    (64, 34, [65536]),               # 1024 candidates, m = 32: the narrowed search at its limit
    (64, 35, [40000]),               # m = 33: the full search on the same chunk count
    (32, 3, [20000, 3000]),          # m = 1
])
def test_select_matches_oracle_register_path(kind, B, K, docs):
    T = sum(docs)
    rows = None if T <= 4096 else np.unique(np.concatenate([
        np.linspace(0, T - 1, 1500).astype(np.int64), np.arange(T - 200, T)]))
    _check(docs, B, K, kind, seed=len(docs) * 1000 + K, rows=rows)


@pytest.mark.parametrize("kind", ["ties", "coarse", "flat", "mixed"])
@pytest.mark.parametrize("B,K,docs,nrows", [
    (16, 32, [24000, 17], 800),      # 1500 candidates: shared-memory staging, 8 warps a CTA
    (16, 64, [320000], 120),         # 20000 candidates: 80 KB a row, 2 warps a CTA
    (16, 30, [320000], 120),         # the same rows, m = 28: narrowed search from shared memory
])
def test_select_matches_oracle_shared_memory_path(kind, B, K, docs, nrows):
    T = sum(docs)
    rows = np.unique(np.concatenate([np.linspace(0, T - 1, nrows).astype(np.int64),
                                     np.arange(T - 40, T), np.arange(docs[0] - 20, docs[0] + 5)]))
    rows = rows[rows < T]
    _check(docs, B, K, kind, seed=7 + K, rows=rows)


def test_select_refuses_rows_past_the_staging_limit_before_launch():
    T, B = 16, 16
    max_seqlen = 16 * (56 * 1024 + 1)  # one block past the limit
    nb = hs.nbmax(max_seqlen, B)
    bs = torch.zeros((T, nb), device="cuda")
    cu = torch.tensor([0, T], device="cuda", dtype=torch.int32)
    with pytest.raises(hs.HSError) as e:
        hs.hs_select_topk(bs, cu, max_seqlen, B, 8)
    assert e.value.status == hs.HS_ERR_UNSUPPORTED
