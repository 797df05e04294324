"""Python wrapper of the CPU oracle for the FP8 (E4M3) 128x128 block-scaled GEMM.

TEST INFRASTRUCTURE ONLY: only the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the CUDA library
and never imports it.  All arithmetic lives in dg_oracle.c (plain C, FP64); this
module only marshals numpy arrays.

Functions and the passages they follow:
  e4m3_table          E4M3 format, demingchina.com/news/60142 §3.1 (format table)
  e4m3_encode         nearest E4M3 value (reading: ties to even code, saturate at 448)
  quantize_blockwise  128x128 block scales from the data range, 2kiu.com/news/5461879
                      §2.1 (block-wise scaling), §3.3 (FP32 scales); scale = amax/448
  gemm_ref            block formula with per-K-block promotion, 2kiu.com/news/5461879
                      §2.1 and §3.3 (FP32 accumulate, segmented accumulation);
                      demingchina.com/news/60142 §3.1 (scales multiplied back at output)
  quantize_groups     one scale per row and 128-element group ("per-group, 128 elements a
                      group", demingchina.com/news/60142 §5.2); otherwise as above
  gemm_ref_rowscale   gemm_ref with those per-row A scales (B keeps 128x128 blocks)
  masked_gemm_ref     masked MoE layout: expert g's first masked_m[g] rows, the dense
                      formula per expert (2kiu.com/news/5461879 §2.2)
  grouped_gemm_ref    experts stored contiguously by expert id, one long matrix
                      (nxmr.cn/news/132300 §2.2), N and K fixed, M varies
                      (2kiu.com/news/5461879 §2.2)
  bf16_from_double    round to nearest BF16, ties to even (reading: the pages say BF16
                      output only)
  check_tolerance     |c - ref| <= 1e-2 |ref| + 1e-3 rms(ref); "<1% relative error vs a
                      higher-precision reference is normal", 2kiu.com/news/5461879 §6
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

BLK = 128

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    from . import build as _build  # noqa: local build of the C oracle
    path = _build.build()
    lib = ctypes.CDLL(path)
    i64 = ctypes.c_int64
    vp = ctypes.c_void_p
    lib.dgo_e4m3_decode.restype = ctypes.c_double
    lib.dgo_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.dgo_e4m3_table.argtypes = [vp]
    lib.dgo_e4m3_encode.restype = ctypes.c_uint8
    lib.dgo_e4m3_encode.argtypes = [ctypes.c_float]
    lib.dgo_e4m3_encode_array.argtypes = [vp, i64, vp]
    lib.dgo_bf16_from_double.restype = ctypes.c_uint16
    lib.dgo_bf16_from_double.argtypes = [ctypes.c_double]
    lib.dgo_bf16_from_double_array.argtypes = [vp, i64, vp]
    lib.dgo_quantize_blockwise.argtypes = [vp, i64, i64, i64, vp, vp]
    lib.dgo_quantize_groups.argtypes = [vp, i64, i64, i64, vp, vp]
    lib.dgo_gemm_ref.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, vp, i64, vp, i64, vp]
    lib.dgo_gemm_ref_rowscale.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, vp, i64, vp, i64, vp]
    lib.dgo_grouped_gemm_ref.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, i64, vp, i64, vp]
    lib.dgo_init()
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def num_threads() -> int:
    """Threads the OpenMP oracle uses (OMP_NUM_THREADS, else all host cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    return int(env) if env else (os.cpu_count() or 1)


# --------------------------------------------------------------------------- E4M3
def e4m3_table() -> np.ndarray:
    """Exact real value of each of the 256 E4M3 codes (NaN at 0x7F and 0xFF)."""
    lib = _load()
    out = np.empty(256, dtype=np.float64)
    lib.dgo_e4m3_table(_ptr(out))
    return out


def e4m3_encode(v) -> np.ndarray:
    """FP32 values -> E4M3 codes (nearest, ties to even code, saturating at 448)."""
    lib = _load()
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib.dgo_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode(q: np.ndarray) -> np.ndarray:
    return e4m3_table()[np.asarray(q, dtype=np.uint8)]


# --------------------------------------------------------------------------- BF16
def bf16_from_double(x) -> np.ndarray:
    """FP64 values -> BF16 bit patterns (uint16), round to nearest, ties to even."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib.dgo_bf16_from_double_array(_ptr(x), x.size, _ptr(out))
    return out


def bf16_bits_to_double(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------- quantize
def quantize_blockwise(x_bf16_bits: np.ndarray):
    """BF16 [R][C] (as uint16 bit patterns) -> (E4M3 codes [R][C], FP32 scales [Rb][Cb])."""
    lib = _load()
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    assert x.ndim == 2
    R, C = x.shape
    Rb, Cb = -(-R // BLK), -(-C // BLK)
    q = np.empty((R, C), dtype=np.uint8)
    s = np.empty((Rb, Cb), dtype=np.float32)
    lib.dgo_quantize_blockwise(_ptr(x), R, C, BLK, _ptr(q), _ptr(s))
    return q, s


def quantize_groups(x_bf16_bits: np.ndarray):
    """BF16 [R][C] -> (E4M3 codes [R][C], FP32 scales [R][Cb]): one scale per row and
    128-column group, s = fl32(amax/448) over the group's elements."""
    lib = _load()
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    assert x.ndim == 2
    R, C = x.shape
    q = np.empty((R, C), dtype=np.uint8)
    s = np.empty((R, -(-C // BLK)), dtype=np.float32)
    lib.dgo_quantize_groups(_ptr(x), R, C, BLK, _ptr(q), _ptr(s))
    return q, s


# --------------------------------------------------------------------------- GEMM
def _idx(a, n):
    if a is None:
        return None, n
    a = np.ascontiguousarray(a, dtype=np.int64)
    return a, a.size


def gemm_ref(A, sA, B, sB, rows=None, cols=None) -> np.ndarray:
    """FP64 block formula for C = A.B^T at the given rows x cols (all if None).

    A [M][K] codes, sA [ceil(M/128)][ceil(K/128)], B [N][K] codes, sB [ceil(N/128)][ceil(K/128)].
    A K that is not a multiple of 128 ends in a partial K block of the columns present.
    """
    lib = _load()
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sA = np.ascontiguousarray(sA, dtype=np.float32)
    sB = np.ascontiguousarray(sB, dtype=np.float32)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2 and K > 0
    assert sA.shape == (-(-M // BLK), -(-K // BLK)) and sB.shape == (-(-N // BLK), -(-K // BLK))
    r, nr = _idx(rows, M)
    c, nc = _idx(cols, N)
    out = np.empty((nr, nc), dtype=np.float64)
    lib.dgo_gemm_ref(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB), M, N, K, BLK,
                     None if r is None else _ptr(r), nr, None if c is None else _ptr(c), nc,
                     _ptr(out))
    return out


def gemm_ref_rowscale(A, sA, B, sB, rows=None, cols=None) -> np.ndarray:
    """gemm_ref with one A scale per row and K block: sA [M][ceil(K/128)]."""
    lib = _load()
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sA = np.ascontiguousarray(sA, dtype=np.float32)
    sB = np.ascontiguousarray(sB, dtype=np.float32)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2 and K > 0
    assert sA.shape == (M, -(-K // BLK)) and sB.shape == (-(-N // BLK), -(-K // BLK))
    r, nr = _idx(rows, M)
    c, nc = _idx(cols, N)
    out = np.empty((nr, nc), dtype=np.float64)
    lib.dgo_gemm_ref_rowscale(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB), M, N, K, BLK,
                              None if r is None else _ptr(r), nr, None if c is None else _ptr(c), nc,
                              _ptr(out))
    return out


def grouped_gemm_ref(A, sA, B, sB, offsets, rows, cols=None) -> np.ndarray:
    """FP64 block formula for the grouped-contiguous layout at the given rows x cols.

    A [M_total][K], sA [M_total/128][ceil(K/128)], B [G][N][K], sB [G][ceil(N/128)][ceil(K/128)],
    offsets int32 [G+1].  Rows owned by no expert come back as NaN.
    """
    lib = _load()
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sA = np.ascontiguousarray(sA, dtype=np.float32)
    sB = np.ascontiguousarray(sB, dtype=np.float32)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    G, N, K = B.shape
    assert off.shape == (G + 1,)
    r, nr = _idx(rows, A.shape[0])
    c, nc = _idx(cols, N)
    out = np.full((nr, nc), np.nan, dtype=np.float64)
    lib.dgo_grouped_gemm_ref(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(off), G, N, K, BLK,
                             _ptr(r), nr, None if c is None else _ptr(c), nc, _ptr(out))
    return out


def masked_gemm_ref(A, sA, B, sB, masked_m, cols=None) -> np.ndarray:
    """FP64 block formula for the masked MoE layout: expert g's first masked_m[g] rows.

    A [G][M_max][K] codes, sA [G][ceil(M_max/128)][ceil(K/128)], B [G][N][K],
    sB [G][ceil(N/128)][ceil(K/128)], masked_m [G] (clamped to [0, M_max]).  Each
    expert is the dense formula on its own slab (2kiu.com/news/5461879 §2.2: only M
    varies between experts).  Rows at or past masked_m[g] come back as NaN.
    """
    A = np.ascontiguousarray(A, dtype=np.uint8)
    G, Mmax, K = A.shape
    N = B.shape[1]
    nc = N if cols is None else len(cols)
    out = np.full((G, Mmax, nc), np.nan, dtype=np.float64)
    for g in range(G):
        m = min(max(int(masked_m[g]), 0), Mmax)
        if m:
            out[g, :m] = gemm_ref(A[g], sA[g], B[g], sB[g], rows=np.arange(m), cols=cols)
    return out


# ----------------------------------------------------------------------- checking
RTOL = 1e-2
ATOL_RMS = 1e-3


def check_tolerance(c: np.ndarray, ref: np.ndarray, rms: float | None = None):
    """Elementwise |c - ref| <= 1e-2 |ref| + 1e-3 rms(ref).

    `rms` is the RMS of ref over all real outputs of the call; when None it is
    taken over `ref` itself.  Returns (ok, n_bad, max_violation_ratio).
    """
    c = np.asarray(c, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if rms is None:
        rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = RTOL * np.abs(ref) + ATOL_RMS * rms
    err = np.abs(c - ref)
    bad = ~(err <= bound)
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if ref.size else 0.0
    return (not bad.any()), int(bad.sum()), ratio
