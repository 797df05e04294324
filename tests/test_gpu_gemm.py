"""GPU parity of the dense block-scaled GEMM against the oracle, element by element.

Small shapes and the 4096^3 workload are compared in full (several tiles and ragged
tails); 8192^3 on one row in every 32-row quarter of every 128-row block (every tile
and every epilogue warp's share of it).  Tolerance: |c - ref| <= 1e-2 |ref| + 1e-3 rms(ref).
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_scales_b200 import binding, inputs

from parity import c_f64, check, dev, oracle_quant, rows_per_quarter, stratified_rms

pytestmark = pytest.mark.gpu


def quantized(d):
    qa, sa = oracle_quant(d.A)
    qb, sb = oracle_quant(d.B)
    return qa, sa, qb, sb


def run(qa, sa, qb, sb, kernel="auto"):
    c = binding.gemm_blockscaled(dev(qa), dev(sa), dev(qb), dev(sb), kernel=kernel)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    return c


SMALL = [(512, 512, 512), (256, 256, 128), (300, 272, 384), (129, 400, 256), (1000, 1008, 640),
         (640, 128, 1024), (200, 16, 128), (384, 144, 2048)]


@pytest.mark.parametrize("M,N,K", SMALL)
@pytest.mark.parametrize("kernel", ["tile", "pair"])
def test_dense_tile_kernels_full_compare(M, N, K, kernel):
    d = inputs.dense_custom(M, N, K, seed=8000 + M + N + K, std_b=0.5)
    qa, sa, qb, sb = quantized(d)
    c = c_f64(run(qa, sa, qb, sb, kernel=kernel))
    ref = oracle.gemm_ref(qa, sa, qb, sb)
    check(c, ref, None, f"{kernel} {M}x{N}x{K}")


SKINNY = [(1, 16, 128), (1, 4096, 4096), (5, 272, 640), (16, 4096, 1024), (17, 512, 512),
          (64, 1040, 768), (100, 256, 256), (128, 4096, 512), (33, 128, 4096)]


@pytest.mark.parametrize("M,N,K", SKINNY)
@pytest.mark.parametrize("kernel", ["skinny", "tile", "pair"])
def test_dense_small_m_all_kernels(M, N, K, kernel):
    d = inputs.dense_custom(M, N, K, seed=8100 + M + N + K)
    qa, sa, qb, sb = quantized(d)
    c = c_f64(run(qa, sa, qb, sb, kernel=kernel))
    ref = oracle.gemm_ref(qa, sa, qb, sb)
    check(c, ref, None, f"{kernel} {M}x{N}x{K}")


KTAIL = [(300, 272, 144), (129, 400, 16), (1000, 1008, 656), (64, 256, 48), (260, 128, 1040),
         (5, 4096, 4000), (128, 512, 4112)]


@pytest.mark.parametrize("M,N,K", KTAIL)
@pytest.mark.parametrize("kernel", ["tile", "pair", "skinny"])
def test_dense_k_tail_all_kernels(M, N, K, kernel):
    """K % 128 != 0: the last K block holds the columns present (TMA zero-fills the rest
    of the box) and is promoted with its own scales."""
    if kernel == "skinny" and M > 128:
        pytest.skip("skinny kernel takes M <= 128")
    d = inputs.dense_custom(M, N, K, seed=8500 + M + N + K)
    qa, sa, qb, sb = quantized(d)
    assert sa.shape[1] == -(-K // 128)
    c = c_f64(run(qa, sa, qb, sb, kernel=kernel))
    check(c, oracle.gemm_ref(qa, sa, qb, sb), None, f"{kernel} {M}x{N}x{K}")


def test_dense_512_workload():
    d = inputs.dense_512()
    qa, sa, qb, sb = quantized(d)
    c = c_f64(run(qa, sa, qb, sb))
    check(c, oracle.gemm_ref(qa, sa, qb, sb), None, "dense 512^3")


def _exact_inputs(M, N, K, seed):
    rng = np.random.default_rng(seed)
    tab = oracle.e4m3_table()
    code_of = {float(tab[c]): c for c in range(0x7F)}
    enc = np.vectorize(lambda x: code_of[abs(float(x))] | (0x80 if x < 0 else 0), otypes=[np.uint8])
    va = rng.choice([-1, 0, 0, 0, 0, 0, 1], size=(M, K))
    vb = rng.choice([-2, -1, 0, 0, 0, 0, 0, 1, 2], size=(N, K))
    sa = (2.0 ** rng.integers(-1, 2, size=(-(-M // 128), -(-K // 128)))).astype(np.float32)
    sb = (2.0 ** rng.integers(-1, 1, size=(-(-N // 128), -(-K // 128)))).astype(np.float32)
    return enc(va), sa, enc(vb), sb


@pytest.mark.parametrize("M,N,K,kernel", [(300, 400, 256, "tile"), (64, 272, 384, "skinny"),
                                          (128, 256, 256, "tile"), (7, 4096, 256, "skinny"),
                                          (300, 400, 256, "pair"), (520, 128, 384, "pair"),
                                          # K tails: the last K block is partial
                                          (300, 400, 208, "pair"), (130, 256, 80, "tile"),
                                          (7, 4096, 176, "skinny")])
def test_dense_exact_small_integers_bit_exact(M, N, K, kernel):
    """Integer E4M3 values and power-of-two scales: every step is exact, so the BF16
    output must equal the oracle's exactly."""
    qa, sa, qb, sb = _exact_inputs(M, N, K, 8200 + M)
    ref = oracle.gemm_ref(qa, sa, qb, sb)
    want = oracle.bf16_bits_to_double(oracle.bf16_from_double(ref))
    assert np.array_equal(want, ref)
    c = c_f64(run(qa, sa, qb, sb, kernel=kernel))
    assert np.array_equal(c, want)


def test_dense_deterministic_and_no_stray_writes():
    M, N, K = 700, 528, 1152
    d = inputs.dense_custom(M, N, K, seed=8300)
    qa, sa, qb, sb = quantized(d)
    A, SA, B, SB = dev(qa), dev(sa), dev(qb), dev(sb)
    guard = 4096
    for kernel in ("tile", "pair"):
        buf = torch.full((M * N + 2 * guard,), -7.0, dtype=torch.bfloat16, device="cuda")
        c = buf[guard:guard + M * N].view(M, N)
        binding.gemm_blockscaled(A, SA, B, SB, C=c, kernel=kernel)
        c2 = binding.gemm_blockscaled(A, SA, B, SB, kernel=kernel)
        torch.cuda.synchronize()
        assert torch.equal(c.view(torch.int16), c2.view(torch.int16))
        assert torch.all(buf[:guard] == -7.0) and torch.all(buf[guard + M * N:] == -7.0)
    c3 = binding.gemm_blockscaled(A[:100], SA[:1], B, SB, kernel="skinny")
    c4 = binding.gemm_blockscaled(A[:100], SA[:1], B, SB, kernel="skinny")
    assert torch.equal(c3.view(torch.int16), c4.view(torch.int16))


def test_dense_unit_scale_identity_invariant():
    """A = identity (E4M3 1.0 on the diagonal), sA = 1: C[m][n] = sB[n/128][m/128] * B[n][m]."""
    M = K = 384
    N = 272
    rng = np.random.default_rng(8400)
    qa = np.zeros((M, K), np.uint8)
    qa[np.arange(M), np.arange(M)] = 0x38
    sa = np.ones((3, 3), np.float32)
    qb = rng.integers(0, 0x7F, size=(N, K)).astype(np.uint8) | (rng.integers(0, 2, (N, K)) << 7).astype(np.uint8)
    sb = (2.0 ** rng.integers(-8, 8, size=(3, 3))).astype(np.float32)
    want = sb[np.arange(N)[None, :] // 128, np.arange(M)[:, None] // 128] * oracle.e4m3_decode(qb).T
    want = oracle.bf16_bits_to_double(oracle.bf16_from_double(want))
    for kernel in ("tile", "pair"):
        c = c_f64(run(qa, sa, qb, sb, kernel=kernel))
        assert np.array_equal(c, want), kernel


# ---------------------------------------------------------------- full-size workloads
def _every_tile_check(d, kernel="auto", seed=0):
    """One row in every 32-row quarter of every 128-row block, all columns, plus the
    outlier rows and the edges: every tile (and each epilogue warp's share of it) of
    the persistent schedule, whichever wave or raster group it fell in, is compared."""
    qa, sa, qb, sb = quantized(d)
    c = c_f64(run(qa, sa, qb, sb, kernel=kernel))
    rng = np.random.default_rng(seed)
    picks = []
    for b in range(0, d.M, 128):
        picks += rows_per_quarter(b, d.M - b, rng)
    special = set(d.outliers.tolist())
    rows = np.unique(np.concatenate([picks, list(special), [0, d.M - 1]]).astype(np.int64))
    ref = oracle.gemm_ref(qa, sa, qb, sb, rows=rows)
    is_out = np.isin(rows, d.outliers)
    w = np.where(is_out, len(special) / max(is_out.sum(), 1), (d.M - len(special)) / max((~is_out).sum(), 1))
    rms = stratified_rms(ref, w)
    return check(c[rows], ref, rms, d.name)


def test_dense_past_one_raster_group():
    """36 m-blocks: a whole raster group of 32 m-blocks, then a partial one of 4, and a
    ragged last block; every tile compared."""
    _every_tile_check(inputs.dense_custom(4500, 768, 384, seed=8800))


def test_dense_4096_outliers_workload():
    """The headline workload compared in full: all 4096 x 4096 outputs."""
    d = inputs.dense_4096_outliers()
    qa, sa, qb, sb = quantized(d)
    c = c_f64(run(qa, sa, qb, sb))
    check(c, oracle.gemm_ref(qa, sa, qb, sb), None, d.name)


@pytest.mark.parametrize("M", [1, 16, 64, 128])
def test_skinny_workload(M):
    d = inputs.skinny(M)
    qa, sa, qb, sb = quantized(d)
    c = c_f64(run(qa, sa, qb, sb))
    ref = oracle.gemm_ref(qa, sa, qb, sb)
    check(c, ref, None, d.name)


@pytest.mark.slow
def test_dense_8192_workload():
    _every_tile_check(inputs.dense_8192())


@pytest.mark.parametrize("M,N,K,kernel", [(512, 768, 1024, "pair"), (512, 768, 1024, "tile"),
                                          (64, 1024, 2048, "skinny")])
def test_per_tensor_special_case_matches_cublaslt(M, N, K, kernel):
    """All A scales equal and all B scales equal: the method is then per-tensor-scaled FP8
    GEMM, which cuBLASLt computes (torch._scaled_mm, a library routine).  A cross-check of
    the whole harness: our kernel, cuBLASLt and the oracle must agree within tolerance."""
    d = inputs.dense_custom(M, N, K, seed=8600 + M + N + K)
    qa, _ = oracle_quant(d.A)
    qb, _ = oracle_quant(d.B)
    a_s, b_s = np.float32(0.0137), np.float32(0.00211)
    sa = np.full((-(-M // 128), K // 128), a_s, np.float32)
    sb = np.full((-(-N // 128), K // 128), b_s, np.float32)
    c = c_f64(run(qa, sa, qb, sb, kernel=kernel))
    A8 = dev(qa).view(torch.float8_e4m3fn)
    B8 = dev(qb).view(torch.float8_e4m3fn)
    c_lt = torch._scaled_mm(A8, B8.t(), scale_a=torch.tensor(float(a_s), device="cuda"),
                            scale_b=torch.tensor(float(b_s), device="cuda"), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    ref = oracle.gemm_ref(qa, sa, qb, sb)
    check(c, ref, None, f"{kernel} per-tensor vs oracle")
    check(c_f64(c_lt), ref, None, "cuBLASLt per-tensor vs oracle")
    rms = float(np.sqrt(np.mean(ref ** 2)))
    check(c, c_f64(c_lt), rms, f"{kernel} vs cuBLASLt")
