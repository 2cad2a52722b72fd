"""Single-GPU FP8 Mixture-of-Experts expert layer for NVIDIA B200 (sm_100a).

The compute lives in libmoe_fp8.so (hand-written CUDA kernels behind the C ABI
declared in include/moe_fp8.h); `api` is a thin ctypes binding with the same
names, and `inputs` draws seeded synthetic workloads."""
