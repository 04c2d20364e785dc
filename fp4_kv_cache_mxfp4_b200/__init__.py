"""CSA2 sparse attention over an FP4 main-KV cache, native to NVIDIA B200.

The compute path is libcsa2.so (C ABI in include/csa2.h, CUDA kernels for
sm_100a in csrc/); ``csa2`` is its Python binding and ``workloads`` draws
the seeded synthetic inputs.
"""
