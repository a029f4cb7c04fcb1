"""Fused GEMM + epilogue for B200 (sm_100a): Python binding over the C ABI.

The binding (``gemm_epilogues_tcgen05_b200.binding``) is loaded on first use,
so that ``synth`` (the seeded input generator) imports without the CUDA
library. Every compute call goes through ``libgemm_epi.so``; there is no
fallback.
"""
