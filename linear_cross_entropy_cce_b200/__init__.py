"""B200-native Cut Cross-Entropy: the classifier matmul fused with
cross-entropy over a large vocabulary, forward and backward, without ever
writing the [N, V] logit matrix to GPU memory.

The compute runs in ``libcce.so`` (hand-written sm_100a CUDA kernels behind a
C ABI, declared in ``include/cce.h``); ``cce`` is the thin ctypes binding.
"""
__all__ = ["cce", "synthetic"]
