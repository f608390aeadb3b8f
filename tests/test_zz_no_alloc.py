"""hs_block_score_static: block scoring for callers that cannot allocate.

Some callers cannot allocate device memory (no allocator is allowed in their
launch path, or their memory is fixed up front), so they cannot hand
hs_block_score a workspace.  hs_block_score_static takes its scratch from a
fixed array inside the library instead.  These tests call it through the C
ABI, twice in a row on different inputs, and compare each result with
hs_block_score's on the same input bit for bit (both run the same
deterministic kernel, so any difference, however small, would mean stale
scratch from the previous call leaking in); and they check that a problem
too large for the fixed array is refused before any device work.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""

import pytest
import torch

from block_sparse_mqa_b200 import hs, synth

pytestmark = pytest.mark.gpu


def _compare(inp, B):
    lse0, bs0, bl0 = hs.hs_block_score(inp.q, inp.k, inp.cu_seqlens, inp.max_seqlen, B,
                                       want_block_lse=True)
    lse1, bs1, bl1 = hs.hs_block_score_static(inp.q, inp.k, inp.cu_seqlens, inp.max_seqlen, B,
                                              want_block_lse=True)
    torch.cuda.synchronize()
    hs.poll_status()
    assert hs.last_path() == hs.HS_PATH_TCGEN05
    assert torch.equal(lse1, lse0)
    assert torch.equal(bl1, bl0)
    assert torch.equal(bs1, bs0)


def test_static_scratch_matches_workspace_entry_point_twice():
    a = synth.make_inputs(900, 64, 576, 512, dtype=torch.bfloat16, seed=21, device="cuda",
                          doc_lengths=[900])
    b = synth.make_inputs(700, 64, 576, 512, dtype=torch.bfloat16, seed=22, device="cuda",
                          doc_lengths=[300, 257, 143])
    assert hs.path(hs.HS_OP_BLOCK_SCORE, torch.bfloat16, 64, 576, 512, 64) == hs.HS_PATH_TCGEN05
    _compare(a, 64)
    _compare(b, 16)  # second call: the scratch still holds the first call's values


def test_static_scratch_refuses_oversized_problem():
    T, H, dk, B = 16384, 32, 192, 16
    need = hs.workspace_size(hs.HS_OP_BLOCK_SCORE, T, 1, T, H, dk, 0, torch.bfloat16, B)
    assert need > 16 << 20
    inp = synth.make_inputs(T, H, dk, 64, dtype=torch.bfloat16, seed=23, device="cuda")
    with pytest.raises(hs.HSError) as e:
        hs.hs_block_score_static(inp.q, inp.k, inp.cu_seqlens, T, B)
    assert e.value.status == hs.HS_ERR_WORKSPACE
    assert "static scratch" in str(e.value)
