"""The GPU tests' helpers that pick rows and compute references, checked on the CPU."""
import numpy as np

import oracle
from fp8_block_scaled_scales_b200 import inputs

from parity import grouped_ref_rows, oracle_quant, rows_per_quarter


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
