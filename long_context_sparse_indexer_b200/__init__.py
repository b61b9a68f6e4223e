"""LSA (LongCat Sparse Attention) hot path for NVIDIA B200 (sm_100a).

``lsa`` binds the C ABI of ``include/lsa.h`` (indexer scores, HI block keys / scores,
top-k with sinks and the SI window, sparse attention with split-KV merge, and the fused
decode step).  All computation runs in the in-tree CUDA library ``_lsa.so``; there is
no CPU path.  Build it with ``python -m long_context_sparse_indexer_b200.build``.
"""
