"""block_sparse_mqa_b200: the HySparse MQA sparse-attention forward path on
B200 (sm_100a).

* ``hs``        ctypes binding of libhs.so (include/hs.h): hs_block_score,
                hs_select_topk, hs_sparse_mqa_fwd, hs_swa_mqa_fwd.
* ``synth``     seeded synthetic inputs.
* ``workloads`` the benchmark / parity workloads.
* ``build``     compiles libhs.so in-tree for sm_100a.
"""

__version__ = "0.3.0"  # = hs_version() of libhs.so (major.minor.patch)
