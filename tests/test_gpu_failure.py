"""Failure detection on the GPU without a GPU fault: a bounded pipeline wait
that nothing completes must give up, report HS_ERR_TIMEOUT through the
status word, and leave the context usable."""

import pytest
import torch

from block_sparse_mqa_b200 import hs, synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    hs.poll_status()  # clean start
    hs.selftest_wait(2_000_000)  # 2 ms limit on a barrier nobody arrives at
    with pytest.raises(hs.HSError) as e:
        hs.poll_status()
    assert e.value.status == hs.HS_ERR_TIMEOUT
    hs.poll_status()  # the status word was cleared
    # the context still runs real work
    inp = synth.make_inputs(130, 64, 576, 512, dtype=torch.bfloat16, seed=1, device="cuda")
    lse, bs, _ = hs.hs_block_score(inp.q, inp.k, inp.cu_seqlens, 130, 64)
    torch.cuda.synchronize()
    hs.poll_status()
    assert torch.isfinite(lse).all()
