"""B200-native MiniMax-M3 block-sparse attention over a paged KV cache.

The compute lives in ``libmsa.so`` (hand-written sm_100a CUDA kernels behind a C ABI,
declared in ``include/msa.h``).  ``block_sparse_paged_scores_b200.msa`` is the thin ctypes
binding; ``workload`` draws seeded synthetic inputs.  Importing this package does not load
the CUDA library; the first call into ``msa`` does, and fails loudly if it is missing.
"""
