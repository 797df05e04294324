"""Property tests of the oracle over random shapes (hypothesis): invariants the block
formula must keep whatever the sizes, ragged tails and zero experts included."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle

from test_oracle_pins import random_finite_codes, random_scales

SETTINGS = settings(max_examples=25, deadline=None)


@SETTINGS
@given(M=st.integers(1, 200), N=st.integers(1, 200), kb=st.integers(1, 3), tail=st.sampled_from([0, 16, 48]),
       seed=st.integers(0, 2 ** 31 - 1))
def test_kblock_permutation_with_scales_is_invariant(M, N, kb, tail, seed):
    """Reordering whole K blocks together with their scale columns changes only the FP64
    summation order of the promoted partials."""
    rng = np.random.default_rng(seed)
    K = 128 * kb + tail
    Kb = -(-K // 128)
    A, B = random_finite_codes(rng, (M, K)), random_finite_codes(rng, (N, K))
    sA, sB = random_scales(rng, (-(-M // 128), Kb)), random_scales(rng, (-(-N // 128), Kb))
    ref = oracle.gemm_ref(A, sA, B, sB)
    if tail:  # keep the partial block last; permute the full ones
        perm = np.concatenate([rng.permutation(Kb - 1), [Kb - 1]])
    else:
        perm = rng.permutation(Kb)
    cols = np.concatenate([np.arange(128 * p, min(K, 128 * p + 128)) for p in perm])
    got = oracle.gemm_ref(np.ascontiguousarray(A[:, cols]), np.ascontiguousarray(sA[:, perm]),
                          np.ascontiguousarray(B[:, cols]), np.ascontiguousarray(sB[:, perm]))
    # FP64 reordering of Kb exact terms moves the sum by at most Kb ulps of sum|term|; bound
    # sum|term| by Kb times the largest a term can be, so the bound holds under any cancellation
    term_max = float(sA.max()) * float(sB.max()) * 128 * 448.0 ** 2
    assert np.all(np.abs(got - ref) <= Kb * Kb * 2.0 ** -52 * term_max)


@SETTINGS
@given(counts=st.lists(st.integers(0, 300), min_size=1, max_size=5), seed=st.integers(0, 2 ** 31 - 1))
def test_grouped_equals_dense_per_expert(counts, seed):
    rng = np.random.default_rng(seed)
    G, N, K = len(counts), 144, 256
    padded = (np.array(counts) + 127) // 128 * 128
    off = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    Mt = int(off[-1])
    A = np.zeros((max(Mt, 1), K), np.uint8)
    A[:Mt] = random_finite_codes(rng, (Mt, K))
    sA = random_scales(rng, (max(Mt, 1) // 128 or 1, 2))
    B, sB = random_finite_codes(rng, (G, N, K)), random_scales(rng, (G, 2, 2))
    rows = np.arange(Mt, dtype=np.int64)
    got = oracle.grouped_gemm_ref(A, sA, B, sB, off, rows)
    for g in range(G):
        sl = slice(off[g], off[g + 1])
        if off[g + 1] > off[g]:
            want = oracle.gemm_ref(A, sA, B[g], sB[g], rows=rows[sl])
            assert np.array_equal(got[sl], want)


@SETTINGS
@given(R=st.integers(1, 300), C=st.sampled_from([16, 112, 128, 144, 400]), scale=st.floats(1e-6, 1e4),
       seed=st.integers(0, 2 ** 31 - 1))
def test_quantizers_round_trip_within_half_a_code(R, C, scale, seed):
    """|dec(q) * s - x| <= half the E4M3 spacing at |x|/s, for both block shapes."""
    import torch
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn((R, C), generator=g) * scale).to(torch.bfloat16)
    bits = x.contiguous().view(torch.int16).numpy().view(np.uint16)
    xv = x.to(torch.float64).numpy()
    tab = oracle.e4m3_table()[:0x7F]
    for q, s, rows in ((*oracle.quantize_blockwise(bits), 128), (*oracle.quantize_groups(bits), 1)):
        sc = s[np.arange(R)[:, None] // rows, np.arange(C)[None, :] // 128].astype(np.float64)
        v = np.abs(xv) / sc
        assert np.all(v <= 448.0 * (1 + 2.0 ** -22))
        idx = np.clip(np.searchsorted(tab, v), 1, 126)
        spacing = tab[idx] - tab[idx - 1]
        err = np.abs(oracle.e4m3_decode(q) * sc - xv) / sc
        assert np.all(err <= 0.5 * spacing * (1 + 1e-6) + 1e-12)
