"""Thin Python binding of libdg.so (argument marshalling only).

Every step of the computation runs in the library's CUDA kernels; this module only
passes device pointers, sizes and the current CUDA stream through the C ABI
declared in include/dg.h, and allocates outputs with torch when the caller did not
pass them.  There is no fallback: if libdg.so is missing or the device is not
sm_100a, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")

DG_OK = 0
STATUS_NAMES = {0: "DG_OK", 1: "DG_ERR_INVALID_ARG", 2: "DG_ERR_SHAPE", 3: "DG_ERR_ALIGNMENT",
                4: "DG_ERR_UNSUPPORTED_DEVICE", 5: "DG_ERR_CUDA", 6: "DG_ERR_TIMEOUT",
                7: "DG_ERR_GROUP_OFFSETS"}
KERNELS = {"auto": 0, "tile": 1, "skinny": 2, "pair": 3, "fused": 4}

# every symbol include/dg.h declares
EXPORTS = ("dg_quantize_blockwise", "dg_quantize_blockwise_masked", "dg_fp8_gemm_blockscaled",
           "dg_fp8_gemm_blockscaled_bf16a",
           "dg_fp8_gemm_blockscaled_bf16a_select",
           "dg_fp8_grouped_gemm_contiguous", "dg_fp8_grouped_gemm_masked", "dg_quantize_1x128",
           "dg_fp8_gemm_1x128", "dg_fp8_gemm_1x128_select",
           "dg_fp8_gemm_blockscaled_select", "dg_status_string", "dg_get_last_device_status",
           "dg_version", "dg_test_set_kernel_control")


class DGError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libdg.so once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                           "`python -m fp8_block_scaled_scales_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.dg_quantize_blockwise.argtypes = [vp, i64, i64, vp, vp, vp]
    L.dg_quantize_blockwise_masked.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp]
    L.dg_fp8_gemm_blockscaled.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.dg_fp8_gemm_blockscaled_select.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, vp]
    L.dg_fp8_gemm_blockscaled_bf16a.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.dg_fp8_gemm_blockscaled_bf16a_select.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, vp]
    L.dg_fp8_grouped_gemm_contiguous.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i64, i64, vp]
    L.dg_fp8_grouped_gemm_masked.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i64, i64, vp]
    L.dg_quantize_1x128.argtypes = [vp, i64, i64, vp, vp, vp]
    L.dg_fp8_gemm_1x128.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.dg_fp8_gemm_1x128_select.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, vp]
    for f in ("dg_quantize_blockwise", "dg_quantize_blockwise_masked", "dg_fp8_gemm_blockscaled",
              "dg_fp8_gemm_blockscaled_select",
              "dg_fp8_gemm_blockscaled_bf16a", "dg_fp8_gemm_blockscaled_bf16a_select",
              "dg_fp8_grouped_gemm_contiguous", "dg_fp8_grouped_gemm_masked", "dg_get_last_device_status",
              "dg_quantize_1x128", "dg_fp8_gemm_1x128", "dg_fp8_gemm_1x128_select"):
        getattr(L, f).restype = ctypes.c_int
    L.dg_get_last_device_status.argtypes = [vp]
    L.dg_status_string.restype = ctypes.c_char_p
    L.dg_status_string.argtypes = [ctypes.c_int]
    L.dg_version.restype = ctypes.c_int
    L.dg_version.argtypes = []
    L.dg_test_set_kernel_control.restype = None
    L.dg_test_set_kernel_control.argtypes = [ctypes.c_uint64, ctypes.c_int]
    _lib = L
    return L


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _p(t: torch.Tensor | None) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_cuda:
        raise ValueError("tensors must be CUDA device tensors")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous (row-major)")
    return ctypes.c_void_p(t.data_ptr())


def _check(status: int, what: str):
    if status != DG_OK:
        raise DGError(status, what)


def _u8(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t


def quantize_blockwise(x: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None,
                       stream=None):
    """BF16 [R][C] -> (E4M3 codes uint8 [R][C], FP32 scales [ceil(R/128)][ceil(C/128)])."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bfloat16 tensor")
    R, C = x.shape
    if q is None:
        q = torch.empty((R, C), dtype=torch.uint8, device=x.device)
    if s is None:
        s = torch.empty(((R + 127) // 128, (C + 127) // 128), dtype=torch.float32, device=x.device)
    _check(lib().dg_quantize_blockwise(_p(x), R, C, _p(_u8(q)), _p(s), _stream(stream)),
           "dg_quantize_blockwise")
    return q, s


def quantize_blockwise_masked(x, masked_m, q=None, s=None, stream=None):
    """Block quantization of masked-MoE activations x [G][M_max][K] (bf16): the first
    masked_m[g] rows of slab g (int32 [G] on the device) as quantize_blockwise would
    quantize them alone; rows past the count and the blocks past the last token are
    neither read nor written."""
    G, M_max, K = x.shape
    if q is None:
        q = torch.zeros((G, M_max, K), dtype=torch.uint8, device=x.device)
    if s is None:
        s = torch.zeros((G, (M_max + 127) // 128, (K + 127) // 128), dtype=torch.float32, device=x.device)
    _check(lib().dg_quantize_blockwise_masked(_p(x), G, M_max, K, _p(masked_m), _p(_u8(q)), _p(s), _stream(stream)),
           "dg_quantize_blockwise_masked")
    return q, s


def gemm_blockscaled(A, sA, B, sB, C=None, kernel: str = "auto", stream=None):
    """C[M][N] (bf16) = block-scaled A[M][K] . B[N][K]^T."""
    A, B = _u8(A), _u8(B)
    M, K = A.shape
    N = B.shape[0]
    if C is None:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _check(lib().dg_fp8_gemm_blockscaled_select(_p(A), _p(sA), _p(B), _p(sB), _p(C), M, N, K,
                                                KERNELS[kernel], _stream(stream)),
           "dg_fp8_gemm_blockscaled")
    return C


def gemm_blockscaled_bf16a(A, B, sB, C=None, QA=None, sA=None, kernel: str = "auto", stream=None):
    """C[M][N] (bf16) = quantize(A)[M][K] . B[N][K]^T from BF16 activations A.

    Returns (C, QA, sA): A's E4M3 codes and 128x128 block scales are outputs too.
    kernel="fused" (M <= 16) quantizes A inside the skinny GEMM, in one launch."""
    M, K = A.shape
    B = _u8(B)
    N = B.shape[0]
    dev = A.device
    if C is None:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if QA is None:
        QA = torch.empty((M, K), dtype=torch.uint8, device=dev)
    if sA is None:
        sA = torch.empty(((M + 127) // 128, (K + 127) // 128), dtype=torch.float32, device=dev)
    _check(lib().dg_fp8_gemm_blockscaled_bf16a_select(_p(A), _p(B), _p(sB), _p(C), _p(_u8(QA)), _p(sA), M, N, K,
                                                      KERNELS[kernel], _stream(stream)),
           "dg_fp8_gemm_blockscaled_bf16a")
    return C, QA, sA


def grouped_gemm_contiguous(A, sA, B, sB, offsets, C=None, stream=None):
    """Grouped-contiguous MoE GEMM: A [M_cap][K], B [G][N][K], offsets int32 [G+1] (device)."""
    A, B = _u8(A), _u8(B)
    Mcap, K = A.shape
    G, N, _ = B.shape
    if C is None:
        C = torch.empty((Mcap, N), dtype=torch.bfloat16, device=A.device)
    _check(lib().dg_fp8_grouped_gemm_contiguous(_p(A), _p(sA), _p(B), _p(sB), _p(C), _p(offsets), Mcap, G,
                                                N, K, _stream(stream)),
           "dg_fp8_grouped_gemm_contiguous")
    return C


def quantize_1x128(x: torch.Tensor, q: torch.Tensor | None = None, s_t: torch.Tensor | None = None,
                   stream=None):
    """BF16 [R][C] -> (E4M3 codes [R][C], FP32 scales [ceil(C/128)][R]), one per row and group."""
    R, C = x.shape
    if q is None:
        q = torch.empty((R, C), dtype=torch.uint8, device=x.device)
    if s_t is None:
        s_t = torch.empty(((C + 127) // 128, R), dtype=torch.float32, device=x.device)
    _check(lib().dg_quantize_1x128(_p(x), R, C, _p(_u8(q)), _p(s_t), _stream(stream)), "dg_quantize_1x128")
    return q, s_t


def gemm_1x128(A, sA_t, B, sB, C=None, kernel: str = "auto", stream=None):
    """C[M][N] (bf16) from A with per-token scales sA_t [ceil(K/128)][M] and 128x128 B scales."""
    A, B = _u8(A), _u8(B)
    M, K = A.shape
    N = B.shape[0]
    if C is None:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _check(lib().dg_fp8_gemm_1x128_select(_p(A), _p(sA_t), _p(B), _p(sB), _p(C), M, N, K, KERNELS[kernel],
                                          _stream(stream)),
           "dg_fp8_gemm_1x128")
    return C


def grouped_gemm_masked(A, sA, B, sB, masked_m, C=None, stream=None):
    """Masked MoE GEMM: A [G][M_max][K], B [G][N][K], masked_m int32 [G] (device).

    Rows at or past masked_m[g] of C are not written (a new C is zero-filled)."""
    A, B = _u8(A), _u8(B)
    G, Mmax, K = A.shape
    N = B.shape[1]
    if C is None:
        C = torch.zeros((G, Mmax, N), dtype=torch.bfloat16, device=A.device)
    _check(lib().dg_fp8_grouped_gemm_masked(_p(A), _p(sA), _p(B), _p(sB), _p(C), _p(masked_m), G, Mmax, N, K,
                                            _stream(stream)),
           "dg_fp8_grouped_gemm_masked")
    return C


def last_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the library's device status word."""
    return lib().dg_get_last_device_status(_stream(stream))


def set_kernel_control(timeout_ns: int = 0, debug_flags: int = 0):
    lib().dg_test_set_kernel_control(timeout_ns, debug_flags)


def version() -> int:
    return lib().dg_version()
