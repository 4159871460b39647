"""B200-native HyperAttention forward pass: sortLSH hashing, segmented sort, block-diagonal and
sampled-column attention with a log-space merge, and the recursive causal variant, as hand-written
sm_100a CUDA kernels behind a C ABI (include/hyper_attn.h).

The Python side only marshals arguments: ``binding`` loads the in-tree shared library and raises if it
is missing; nothing here computes any step of the method.
"""
__all__ = ["binding", "workload"]
