"""B200-native Cross-Layer Sparse Attention (CLSA, "You Only Index Once").

The hot path -- indexer scores, exact top-k routing computed once, gather of the
selected K/V rows, and token-sparse GQA attention for every cross-decoder layer --
runs in hand-written sm_100a CUDA kernels behind the C ABI declared in
``include/clsa.h``.  ``long_context_sparse_clsa_b200.clsa`` is the thin Python
binding (argument marshalling only).  Importing this package does not load the
CUDA library; the first call into ``clsa`` does, and fails loudly if the library
is missing.
"""
__all__ = ["inputs", "clsa"]
