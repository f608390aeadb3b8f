"""The HySparse forward workloads, as plain data.

Each entry names a workload by what it is (sizes included).  Shapes follow
the absorbed-MLA MQA layout of "HySparse MQA sparse attention ...",
PaddleFleet pull request 1470, section "FlashMLA sparse kernel
constraints": 64 query heads over one shared KV head, Dk = 512 latent + 64
RoPE, Dv = 512.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

from .synth import packed_doc_lengths


@dataclass(frozen=True)
class Workload:
    name: str
    total_tokens: int
    num_heads: int
    dk: int
    dv: int
    dtype: torch.dtype
    block_size: int
    topk: int
    window: int
    doc_lengths: tuple = field(default=())
    swa_dk: Optional[int] = None      # separate SWA layer dims (sweep)
    swa_dv: Optional[int] = None

    def docs(self) -> list:
        return list(self.doc_lengths) if self.doc_lengths else [self.total_tokens]

    @property
    def max_seqlen(self) -> int:
        return max(self.docs())


def _packed_16k():
    return tuple(packed_doc_lengths(16384, 6, 512, seed=0))


TINY = Workload("tiny_T256_H4_dk64_dv48_f32_B16_k4_w32", 256, 4, 64, 48,
                torch.float32, 16, 4, 32)
MAIN = Workload("mla_T4096_H64_dk576_dv512_bf16_B64_k16_w512", 4096, 64, 576, 512,
                torch.bfloat16, 64, 16, 512)
PACKED = Workload("packed6_T16384_H64_dk576_dv512_bf16_B64_k16_w512", 16384, 64, 576,
                  512, torch.bfloat16, 64, 16, 512, doc_lengths=_packed_16k())
LONG = Workload("long_T65536_H64_dk576_dv512_bf16_B64_k32_w1024", 65536, 64, 576, 512,
                torch.bfloat16, 64, 32, 1024)


def sweep(topk: int) -> Workload:
    """4 documents of 32768 tokens; top-k in {8, 16, 32, 64}."""
    return Workload("sweep_4x32768_H64_dk576_dv512_bf16_B64_k%d" % topk, 131072, 64,
                    576, 512, torch.bfloat16, 64, topk, 1024,
                    doc_lengths=(32768,) * 4)


def sweep_swa(window: int) -> Workload:
    """The separate SWA-only layer of the sweep: Dk 192, Dv 128."""
    return Workload("sweep_swa_4x32768_H64_dk192_dv128_bf16_w%d" % window, 131072, 64,
                    192, 128, torch.bfloat16, 64, 16, window,
                    doc_lengths=(32768,) * 4)


# shape variants of the main workload: no RoPE chunk (Dk = 512) and a latent
# narrower than 512 (Dv = 448), the two widths the FlashMLA constraints and
# the value-padding note name
NOROPE = Workload("mla_T4096_H64_dk512_dv512_bf16_B64_k16_w512", 4096, 64, 512, 512,
                  torch.bfloat16, 64, 16, 512)
NARROW_V = Workload("mla_T4096_H64_dk576_dv448_bf16_B64_k16_w512", 4096, 64, 576, 448,
                    torch.bfloat16, 64, 16, 512)

ALL = {w.name: w for w in [TINY, MAIN, PACKED, LONG, NOROPE, NARROW_V]
       + [sweep(k) for k in (8, 16, 32, 64)]
       + [sweep_swa(w) for w in (256, 1024, 4096)]}
