"""Seeded synthetic inputs for the HySparse MQA forward workloads.

This module only draws random numbers and packs documents; it holds none of
the attention arithmetic.  Both the CUDA tests and the CPU oracle consume
what it returns (the oracle after a lossless cast to float64), so the two
sides always see the same rounded values.

Recipe (the workloads' stated distributions):

* q [T, H, Dk], k [T, Dk], v [T, Dv] ~ N(0, 1), drawn in that order in
  float32 from ``torch.Generator(device).manual_seed(seed)``, then rounded
  to the workload dtype (bf16 round-to-nearest-even, or kept float32);
* sink [H] ~ N(0, 1) float32, drawn after v from the same generator;
* packed documents: n documents of at least ``min_len`` tokens whose
  lengths are ``min_len`` plus the gaps between n - 1 sorted integer cut
  points drawn uniformly from [0, T - n * min_len] by
  ``numpy.random.default_rng(seed)``; they sum to T exactly.

The draws depend on the device's generator (CPU and CUDA streams differ),
so a test always hands the very same tensors to the kernel and the oracle.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


@dataclass
class Inputs:
    q: torch.Tensor            # [T, H, Dk]
    k: torch.Tensor            # [T, Dk]
    v: torch.Tensor            # [T, Dv]
    sink: torch.Tensor         # [H] float32
    cu_seqlens: torch.Tensor   # [num_docs + 1] int32 (same device as q)
    max_seqlen: int
    meta: dict = field(default_factory=dict)

    @property
    def total_tokens(self) -> int:
        return int(self.q.shape[0])


def packed_doc_lengths(total: int, num_docs: int, min_len: int, seed: int):
    """Document lengths >= min_len that sum to ``total`` (see module doc)."""
    if num_docs < 1 or total < num_docs * min_len:
        raise ValueError("cannot pack %d docs of >= %d tokens into %d"
                         % (num_docs, min_len, total))
    rng = np.random.default_rng(seed)
    free = total - num_docs * min_len
    cuts = np.sort(rng.integers(0, free + 1, size=num_docs - 1))
    edges = np.concatenate([[0], cuts, [free]])
    lengths = min_len + np.diff(edges)
    assert int(lengths.sum()) == total
    return [int(x) for x in lengths]


def cu_from_lengths(lengths) -> list[int]:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return cu


def make_inputs(total_tokens: int, num_heads: int, dk: int, dv: int,
                dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                device="cpu", doc_lengths: Optional[list] = None,
                sink_std: float = 1.0) -> Inputs:
    """Draw q, k, v, sink for one workload (see module doc for the recipe).

    ``doc_lengths`` defaults to a single document of ``total_tokens``.
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    f32 = torch.float32
    q = torch.randn((total_tokens, num_heads, dk), generator=g, device=device, dtype=f32)
    k = torch.randn((total_tokens, dk), generator=g, device=device, dtype=f32)
    v = torch.randn((total_tokens, dv), generator=g, device=device, dtype=f32)
    sink = torch.randn((num_heads,), generator=g, device=device, dtype=f32) * sink_std
    if dtype != f32:
        q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    if doc_lengths is None:
        doc_lengths = [total_tokens]
    if sum(doc_lengths) != total_tokens:
        raise ValueError("doc lengths must sum to total_tokens")
    cu = cu_from_lengths(doc_lengths)
    cu_t = torch.tensor(cu, dtype=torch.int32, device=device)
    return Inputs(q=q, k=k, v=v, sink=sink, cu_seqlens=cu_t,
                  max_seqlen=max(doc_lengths) if doc_lengths else 0,
                  meta={"seed": seed, "doc_lengths": list(doc_lengths)})


def sample_rows(cu_seqlens, per_doc: int, seed: int = 0) -> np.ndarray:
    """A fixed seeded sample of query rows: ``per_doc`` tokens per document
    spread uniformly over its positions, always including its first and last
    token (sorted, unique)."""
    cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    rng = np.random.default_rng(seed + 7919)
    rows = []
    for bos, eos in zip(cu[:-1], cu[1:]):
        n = eos - bos
        if n == 0:
            continue
        if n <= per_doc:
            rows.extend(range(bos, eos))
            continue
        pick = rng.choice(n, size=per_doc - 2, replace=False)
        rows.extend([bos, eos - 1])
        rows.extend(int(bos + p) for p in pick)
    return np.unique(np.asarray(rows, dtype=np.int64))


def plant_block_order(inp: Inputs, block_size: int, gap: float = 3.0, seed: int = 0,
                      scale: Optional[float] = None, alpha: float = 4.0):
    """Structured copy of ``inp`` whose top-k choice is well separated.

    Each document d gets a seeded random permutation ``perms[d]`` of its key
    blocks (``numpy.random.default_rng(seed + 104729).permutation``, one draw
    per document, in document order).  Feature 0 of every query row is set to
    ``alpha`` and feature 0 of key j (doc-local block b of document d) to
    ``gap * perms[d][b] / (scale * alpha)``, so that a logit
    ``scale * <q, k_j>`` is the other features' random product plus
    ``gap * perms[d][b]`` (up to the rounding of that one key value to the
    input dtype).  With ``gap`` far above the spread of a block's random
    log-mass, every head ranks the complete blocks of a document in
    ``perms[d]`` order.  ``scale`` defaults to Dk^-1/2.  Returns
    ``(inputs, perms)``; the caller's tensors are not modified.
    """
    dk = inp.q.shape[2]
    sc = float(dk) ** -0.5 if scale is None else float(scale)
    cu = [int(x) for x in inp.cu_seqlens.tolist()]
    rng = np.random.default_rng(seed + 104729)
    perms = []
    val = np.zeros(inp.total_tokens, dtype=np.float64)
    for bos, eos in zip(cu[:-1], cu[1:]):
        nb = (eos - bos + block_size - 1) // block_size
        perm = rng.permutation(nb) if nb > 0 else np.zeros(0, dtype=np.int64)
        perms.append(perm)
        for j in range(bos, eos):
            val[j] = gap * float(perm[(j - bos) // block_size]) / (sc * alpha)
    q = inp.q.clone()
    k = inp.k.clone()
    q[:, :, 0] = alpha
    k[:, 0] = torch.as_tensor(val, dtype=torch.float32, device=k.device).to(k.dtype)
    meta = dict(inp.meta)
    meta.update({"planted_gap": gap, "planted_seed": seed, "planted_alpha": alpha})
    return Inputs(q=q, k=k, v=inp.v, sink=inp.sink, cu_seqlens=inp.cu_seqlens,
                  max_seqlen=inp.max_seqlen, meta=meta), perms

