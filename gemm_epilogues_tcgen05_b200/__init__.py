"""Fused GEMM + epilogue for B200 (sm_100a): Python binding over the C ABI.

The binding (``gemm_epilogues_tcgen05_b200.binding``) is loaded on first use,
so that ``synth`` (the seeded input generator) imports without the CUDA
library. Every compute call goes through ``libgemm_epi.so``; there is no
fallback.
"""

from .binding import (BF16, BIAS, DRELU_BGRAD, EPILOGS, F16, RELU_AUX_BIAS, RELU_BIAS, GemmEpiError, Plan,  # noqa: F401
                      gemm_epi_free, gemm_epi_last_error, gemm_epi_plan, lib)
