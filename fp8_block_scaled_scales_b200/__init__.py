"""FP8 (E4M3) 128x128 block-scaled GEMM for B200 (sm_100a).

The compute lives in libdg.so (hand-written CUDA kernels behind a C ABI,
include/dg.h); this package is its Python binding plus the seeded input
generators used by the tests and the benchmark.
"""
from .binding import (DGError, gemm_1x128, gemm_blockscaled, gemm_blockscaled_bf16a,  # noqa: F401
                      grouped_gemm_contiguous, grouped_gemm_masked, last_device_status, quantize_blockwise,
                      quantize_1x128, set_kernel_control, version)
