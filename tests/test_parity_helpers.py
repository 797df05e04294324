"""The GPU tests' helpers that pick rows and compute references, checked on the CPU."""
import numpy as np

import oracle
from fp8_block_scaled_scales_b200 import inputs

from parity import grouped_ref_rows, oracle_quant, oracle_quant_tokens, rows_per_quarter


def test_grouped_ref_rows_equals_the_grouped_oracle_routine():
    w = inputs.grouped_custom(4, 256, 208, [130, 0, 5, 300], seed=31)
    qa, sa = oracle_quant(w.A)
    qb, sb = oracle_quant(w.B)
    rows = np.flatnonzero(inputs.real_row_mask(w.counts, w.offsets))
    want = oracle.grouped_gemm_ref(qa, sa, qb, sb, w.offsets, rows)
    got = grouped_ref_rows(qa, sa, qb, sb, w.offsets, rows)
    assert np.array_equal(got, want)


def test_rows_per_quarter_hits_each_quarter_that_holds_rows():
    rng = np.random.default_rng(0)
    for count in (1, 31, 32, 33, 100, 128, 500):
        rows = rows_per_quarter(256, count, rng)
        assert len(rows) == -(-min(count, 128) // 32)
        for q, r in enumerate(rows):
            assert 256 + 32 * q <= r < 256 + min(32 * q + 32, count)


def test_oracle_quant_tokens_is_the_block_quantizer_on_each_experts_tokens():
    """Per-expert reference for the masked-layout quantizer: slab g's first counts[g] rows
    quantized as a matrix of their own, so the rows past a count (here 100x larger) touch
    neither the codes nor the scales; counts outside [0, M_max] are clamped."""
    w = inputs.masked_custom(3, 256, 128, 272, [77, 0, 256], seed=41)
    qa, sa = oracle_quant_tokens(w.A, [77, -3, 999])
    q0, s0 = oracle.quantize_blockwise(inputs.bf16_bits(w.A[0, :77]))
    assert np.array_equal(qa[0, :77], q0) and np.array_equal(sa[0, :1], s0)
    assert not qa[0, 77:].any() and np.all(sa[0, 1:] == 1.0)
    assert not qa[1].any() and np.all(sa[1] == 1.0)
    q2, s2 = oracle.quantize_blockwise(inputs.bf16_bits(w.A[2]))
    assert np.array_equal(qa[2], q2) and np.array_equal(sa[2], s2)
    # the whole-slab quantization differs: its first block's amax sees the large rows
    qw, sw = oracle.quantize_blockwise(inputs.bf16_bits(w.A[0]))
    assert sw[0, 0] > s0[0, 0]
