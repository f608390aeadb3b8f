"""CPU oracle for the HySparse MQA forward path (test infrastructure only).

This package is the plain, slow, float64 definition of the four forward steps
(block scoring, top-k block selection, block-sparse MQA attention and
sliding-window MQA attention), of the full layer's forward that emits the
block scores with its attention output, of the SWA layer that combines the
window branch with the sparse branch on the shared KV, and of the backward
of the two attention steps, which the CUDA library is checked against.

It is test infrastructure: only the test-suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it.
The CUDA product path never imports it and shares no code with it.

Modules
-------
hysparse
    Vectorised NumPy float64 implementation of the four steps, of the full
    layer's fused forward (``full_layer_fwd``) and of the SWA layer's two
    branches combined (``swa_layer_fwd``).
backward
    The gradient of the two attention steps (dq, dk, dv, sink gradient).
loops
    Pure-Python loop restatements, for brute-force checks on tiny inputs.

Parity status: every function here is pinned by a test under ``tests/``
(closed forms, library special cases, brute force, invariants); none is
"parity unpinned".
"""

from .hysparse import (  # noqa: F401
    doc_bounds,
    block_score,
    select_topk,
    sparse_key_set,
    window_key_set,
    attend,
    sparse_mqa_fwd,
    swa_mqa_fwd,
    dense_causal_fwd,
    full_layer_fwd,
    swa_layer_fwd,
)
