"""GPU parity of per-token (1 x 128 group) activation scales: the group quantizer and
the GEMM that promotes each row with its own scale."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_scales_b200 import binding, inputs

from parity import c_f64, check, dev

pytestmark = pytest.mark.gpu


def oracle_groups(x_bf16):
    return oracle.quantize_groups(inputs.bf16_bits(x_bf16))


@pytest.mark.parametrize("R,C", [(1, 16), (130, 384), (300, 1040), (4096, 4096)])
def test_group_quantizer_bit_exact(R, C):
    if (R, C) == (4096, 4096):
        x = inputs.dense_4096_outliers().A
    else:
        x = inputs.dense_custom(R, 16, C, seed=8900 + R + C, outlier_frac=0.02).A
    q, s_t = binding.quantize_1x128(x.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = oracle_groups(x)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s_t.cpu().numpy().T.view(np.uint32), s_ref.view(np.uint32))


def run(qa, sa_rows, qb, sb, kernel):
    sa_t = np.ascontiguousarray(sa_rows.T)
    c = binding.gemm_1x128(dev(qa), dev(sa_t), dev(qb), dev(sb), kernel=kernel)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    return c


SHAPES = [(512, 512, 512), (300, 272, 384), (129, 400, 256), (1000, 1008, 656), (640, 128, 1024),
          (7, 4096, 256), (200, 16, 144)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("kernel", ["tile", "pair"])
def test_rowscale_gemm_full_compare(M, N, K, kernel):
    d = inputs.dense_custom(M, N, K, seed=9100 + M + N + K, outlier_frac=0.02)
    qa, sa = oracle_groups(d.A)
    qb, sb = oracle.quantize_blockwise(inputs.bf16_bits(d.B))
    c = c_f64(run(qa, sa, qb, sb, kernel))
    check(c, oracle.gemm_ref_rowscale(qa, sa, qb, sb), None, f"1x128 {kernel} {M}x{N}x{K}")


@pytest.mark.parametrize("kernel", ["tile", "pair"])
def test_rowscale_exact_small_integers(kernel):
    """Integer values and power-of-two row scales: exact, so bit-equal to the oracle."""
    rng = np.random.default_rng(9200)
    M, N, K = 300, 400, 256  # sparse small integers: every sum fits BF16's 8-bit significand
    tab = oracle.e4m3_table()
    code_of = {float(tab[c]): c for c in range(0x7F)}
    enc = np.vectorize(lambda x: code_of[abs(float(x))] | (0x80 if x < 0 else 0), otypes=[np.uint8])
    qa = enc(rng.choice([-1, 0, 0, 0, 0, 0, 1], size=(M, K)))
    qb = enc(rng.choice([-2, -1, 0, 0, 0, 0, 0, 1, 2], size=(N, K)))
    sa = (2.0 ** rng.integers(-1, 2, size=(M, 2))).astype(np.float32)
    sb = (2.0 ** rng.integers(-1, 1, size=(4, 2))).astype(np.float32)
    ref = oracle.gemm_ref_rowscale(qa, sa, qb, sb)
    want = oracle.bf16_bits_to_double(oracle.bf16_from_double(ref))
    assert np.array_equal(want, ref)
    assert np.array_equal(c_f64(run(qa, sa, qb, sb, kernel)), want)


@pytest.mark.parametrize("kernel", ["tile", "pair"])
def test_rowscale_equals_block_form_when_rows_share_scales(kernel):
    """Row scales that repeat each 128-row block's scale give the block GEMM, bit for bit."""
    d = inputs.dense_custom(520, 512, 768, seed=9300)
    qa, sa_blk = oracle.quantize_blockwise(inputs.bf16_bits(d.A))
    qb, sb = oracle.quantize_blockwise(inputs.bf16_bits(d.B))
    sa_rows = np.ascontiguousarray(sa_blk[np.arange(520) // 128])
    c_rows = run(qa, sa_rows, qb, sb, kernel)
    c_blk = binding.gemm_blockscaled(dev(qa), dev(sa_blk), dev(qb), dev(sb), kernel=kernel)
    torch.cuda.synchronize()
    assert torch.equal(c_rows.view(torch.int16), c_blk.view(torch.int16))


def test_rowscale_full_size_outlier_rows():
    """M=N=K=4096 with 1% outlier rows: per-token scales, sampled rows incl. every outlier."""
    d = inputs.dense_4096_outliers()
    q, s_t = binding.quantize_1x128(d.A.cuda())
    qb, sb = binding.quantize_blockwise(d.B.cuda())
    c = binding.gemm_1x128(q, s_t, qb, sb)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    rows = np.unique(np.concatenate([d.outliers, np.random.default_rng(0).integers(0, 4096, 40), [0, 4095]]))
    qa_h, sa_h = q.cpu().numpy(), np.ascontiguousarray(s_t.cpu().numpy().T)
    ref = oracle.gemm_ref_rowscale(qa_h, sa_h, qb.cpu().numpy(), sb.cpu().numpy(), rows=rows.astype(np.int64))
    check(c_f64(c)[rows], ref, None, "1x128 4096^3 sampled rows")
