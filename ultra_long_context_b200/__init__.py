"""B200-native Hierarchical Sparse Attention (HSA).

The operator (explainer page of "Every Token Counts: Generalizing 16M Ultra-Long Context in Large
Language Models", "How It Works (Technically)") scores each query against one landmark per
completed 64-token chunk, keeps the top-K chunks, runs softmax attention inside each selected chunk
separately and blends the K chunk outputs by the softmax of their retrieval scores.

All arithmetic runs in the CUDA library ``libhsa_b200.so`` (sm_100a) behind the C ABI declared in
``include/hsa.h``; ``ultra_long_context_b200.hsa`` is its Python binding. Importing this package does
not load the library; the first call into ``hsa`` does, and fails loudly if it is missing.
"""
