"""B200-native (sm_100a) LLM.int8() linear layer: outlier-aware mixed-precision
decomposition plus vector-wise int8 matrix multiplication.

The CUDA library (libllmint8.so, C ABI in include/llmint8.h) is loaded lazily
by ``binding``; importing this package alone does not touch the GPU.
"""
__all__ = ["binding", "workloads", "build"]
