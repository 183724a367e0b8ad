"""B200-native (sm_100a) routed MoE layer forward: router softmax top-k, permute into
expert groups, grouped gate/up GEMM with fused SwiGLU, grouped down GEMM, and the
gate-weighted combine -- hand-written CUDA kernels behind a C ABI (``include/moe.h``).

The Python side only marshals arguments (``api``); the native library is loaded
on first use and its absence is an error, never a fallback.
"""
__all__ = ["api", "inputs"]
