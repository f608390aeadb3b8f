"""The algorithmic work the benchmark divides its times by, checked on the
CPU against counts over the oracle's own key sets (no GPU).

The roofline fractions bench.py reports are (algorithmic flops or bytes) /
(kernel time x peak); the counts below are the numerators' only inputs:
valid causal pairs (step 1, the full layer), window pairs (step 4), the
pairs of the selected blocks (step 3) and step 2's bytes (each query reads
the scores of its candidate blocks 0 .. bq and writes topk ids).
"""

import numpy as np
import pytest
import torch

import bench
import oracle.hysparse as O
from block_sparse_mqa_b200 import synth

DOCS = [[1], [5], [64], [100, 0, 37], [130, 1, 65, 64], [257, 3]]


def _bounds(docs):
    cu = synth.cu_from_lengths(docs)
    return [(int(cu[i]), int(cu[i + 1])) for i in range(len(docs))]


@pytest.mark.parametrize("docs", DOCS)
def test_causal_pairs_count_every_key_up_to_the_query(docs):
    brute = sum(len(O.window_key_set(t, bos, eos - bos + 1))
                for bos, eos in _bounds(docs) for t in range(bos, eos))
    assert bench.causal_pairs(docs) == brute


@pytest.mark.parametrize("docs", DOCS)
@pytest.mark.parametrize("W", [1, 3, 64, 1000])
def test_window_pairs_match_the_oracle_window(docs, W):
    brute = sum(len(O.window_key_set(t, bos, W)) for bos, eos in _bounds(docs)
                for t in range(bos, eos))
    assert bench.window_pairs(docs, W) == brute


@pytest.mark.parametrize("docs", DOCS)
@pytest.mark.parametrize("B", [16, 64])
@pytest.mark.parametrize("topk", [1, 4, 16])
def test_select_bytes_count_candidate_scores_and_ids(docs, B, topk):
    reads = sum((t - bos) // B + 1 for bos, eos in _bounds(docs) for t in range(bos, eos))
    assert bench.select_bytes(docs, B, topk) == 4.0 * reads + 4.0 * sum(docs) * topk


@pytest.mark.parametrize("docs,B,K", [([130, 1, 65, 64], 16, 4), ([300], 32, 3),
                                      ([257, 3], 64, 2), ([90, 90], 16, 16)])
def test_sparse_pairs_match_the_oracle_key_sets(docs, B, K):
    T = sum(docs)
    cu = [int(x) for x in synth.cu_from_lengths(docs)]
    nb = max(1, -(-max(docs) // B))
    rng = np.random.default_rng(T + B + K)
    scores = rng.random((T, nb))
    idx = O.select_topk(scores, cu, B, K)
    brute = 0
    for bos, eos in _bounds(docs):
        for t in range(bos, eos):
            brute += len(O.sparse_key_set(t, bos, eos, idx[t], B))
    assert bench.sparse_pairs(torch.as_tensor(idx), cu, B) == brute
