"""Pins for the CPU oracle: each test checks it against something other than itself.

* E4M3 table: torch's float8_e4m3fn decoding (a library routine), the format facts
  printed on the DeepGEMM FP8 write-up (demingchina.com/news/60142 §3.1 table), and
  invariants of the format.
* Encoder: torch's float8_e4m3fn cast (round to nearest even) swept over every FP32
  value in the E4M3 exponent range; closed forms for saturation and underflow.
* BF16 rounding: exact rational rounding in Python integers / Fractions.
* GEMM: exact integer arithmetic (codes x 2^9 are integers, so each K-block partial
  is an exact int64 matmul) with the scale formula summed in Fractions; exact
  small-integer cases; identity / unit-scale / row-doubling / K-block permutation /
  transpose / grouped-equals-dense invariants.
* Quantizer: E4M3 round-trip error bound, the amax element landing on +-448, and a
  cross-check through torch's FP32 division and float8 cast.
"""
from fractions import Fraction
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------- helpers
def torch_decode(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def codes_to_int(codes: np.ndarray) -> np.ndarray:
    """E4M3 code -> value * 2^9 as an exact int64, via torch's decoding."""
    v = torch_decode(codes) * 512.0
    iv = v.astype(np.int64)
    assert np.array_equal(iv.astype(np.float64), v)
    return iv


def random_finite_codes(rng, shape, max_code=0x7E):
    c = rng.integers(0, max_code + 1, size=shape, dtype=np.int64)
    sign = rng.integers(0, 2, size=shape, dtype=np.int64) << 7
    return (c | sign).astype(np.uint8)


def random_scales(rng, shape):
    # positive FP32 scales spread over a few binades, like amax/448 of real data
    return (rng.uniform(0.5, 2.0, size=shape) * 2.0 ** rng.integers(-12, 2, size=shape)).astype(np.float32)


def exact_ref(A, sA, B, sB, with_abs=False, a_rows=128):
    """Exact block formula as Fractions: integer K-block partials, Fraction scale sum.
    A's scale of row m is sA[m // a_rows] (128: 128x128 blocks, 1: one per row).

    With with_abs, also returns sum_kb |s_kb * P_kb| (float), the scale of the FP64
    summation error bound."""
    M, K = A.shape
    N = B.shape[0]
    Kb = -(-K // 128)  # a partial last block holds the K % 128 columns present
    Ai, Bi = codes_to_int(A), codes_to_int(B)
    out = [[Fraction(0)] * N for _ in range(M)]
    absum = np.zeros((M, N))
    parts = []
    for kb in range(Kb):
        sl = slice(128 * kb, 128 * kb + 128)
        parts.append(Ai[:, sl] @ Bi[:, sl].T)  # int64, exact: |sum| < 2^45
    fa = [[Fraction(float(x)) for x in row] for row in sA]
    fb = [[Fraction(float(x)) for x in row] for row in sB]
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for kb in range(Kb):
                t = fa[m // a_rows][kb] * fb[n // 128][kb] * int(parts[kb][m, n])
                acc += t
                absum[m, n] += abs(float(t)) / 2.0 ** 18
            out[m][n] = acc / (1 << 18)
    return (out, absum) if with_abs else out


def bf16_round_exact(x: Fraction) -> float:
    """Nearest BF16 to a rational, ties to even, by integer arithmetic."""
    if x == 0:
        return 0.0
    sign = -1.0 if x < 0 else 1.0
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** max(e - 7, -133)
    r = a / q
    fl = r.numerator // r.denominator
    frac = r - fl
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * float(fl * q)


def bits_to_f64(h):
    return oracle.bf16_bits_to_double(np.asarray(h, dtype=np.uint16))


# ------------------------------------------------------------------ E4M3 table
def test_e4m3_table_matches_torch_decode():
    tab = oracle.e4m3_table()
    ref = torch_decode(np.arange(256, dtype=np.uint8))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(tab), nan)
    assert np.array_equal(tab[~nan], ref[~nan])
    # the sign of zero
    assert np.signbit(tab[0x80]) and not np.signbit(tab[0x00])


def test_e4m3_table_invariants_and_golden():
    tab = oracle.e4m3_table()
    assert np.isnan(tab[0x7F]) and np.isnan(tab[0xFF])
    assert np.count_nonzero(np.isfinite(tab)) == 254
    pos = tab[:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(tab[0x80:0xFF], -pos)
    assert pos[1] == 2.0 ** -9 and pos[8] == 2.0 ** -6
    # every finite value is a multiple of 2^-9 (used by the exactness argument)
    assert np.all(np.mod(pos * 512.0, 1.0) == 0.0)
    # format facts printed on the page
    with open(os.path.join(GOLDEN, "e4m3_format.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    e4m3 = [r for r in rows if r[0] == "E4M3"][0]
    sign_bits, exp_bits, man_bits, vmax = int(e4m3[1]), int(e4m3[2]), int(e4m3[3]), float(e4m3[4])
    assert sign_bits + exp_bits + man_bits == 8
    assert np.nanmax(tab) == vmax
    # 2^exp_bits exponent codes x 2^man_bits mantissas per sign, minus the NaN code
    assert np.count_nonzero(np.isfinite(tab[:128])) == 2 ** (exp_bits + man_bits) - 1


# --------------------------------------------------------------------- encoder
def test_encoder_exhaustive_against_torch_cast():
    """Every FP32 value with 2^-12 <= |v| < 2^9 (and below 464) against torch's cast."""
    lane = np.arange(1 << 23, dtype=np.uint32)
    for sign in (0, 1):
        for bexp in range(127 - 12, 127 + 9):
            bits = lane | np.uint32(bexp << 23) | np.uint32(sign << 31)
            v = bits.view(np.float32)
            v = v[np.abs(v) < 464.0]
            got = oracle.e4m3_encode(v)
            want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            bad = np.flatnonzero(got != want)
            assert bad.size == 0, (sign, bexp, v[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_encoder_small_and_saturating_closed_forms():
    rng = np.random.default_rng(7)
    # below half the smallest subnormal (2^-10) everything rounds to a signed zero,
    # and exactly 2^-10 is a tie that goes to the even code 0
    tiny = np.concatenate([rng.uniform(0, 2.0 ** -10, 100000), [2.0 ** -10, 1e-45, 0.0]]).astype(np.float32)
    assert np.all(oracle.e4m3_encode(tiny) == 0x00)
    assert np.all(oracle.e4m3_encode(-tiny) == 0x80)
    # satfinite: anything at or beyond 448 (infinity included) clamps to +-448
    big = np.concatenate([rng.uniform(448, 1e6, 100000), [448.0, 464.0, 3e38, np.inf]]).astype(np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)
    # random values across the whole float range agree with torch below 464
    bits = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) < 464)]
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), want)


def test_encoder_ties_go_to_even_code():
    tab = oracle.e4m3_table()[:0x7F]
    mids = ((tab[:-1] + tab[1:]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (tab[:-1] + tab[1:]) / 2)  # exact in FP32
    got = oracle.e4m3_encode(mids).astype(np.int64)
    lo = np.arange(126)
    assert np.all(got == np.where(lo % 2 == 0, lo, lo + 1))
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(0))
    assert np.array_equal(oracle.e4m3_encode(up).astype(np.int64), lo + 1)
    assert np.array_equal(oracle.e4m3_encode(dn).astype(np.int64), lo)


# ----------------------------------------------------------------------- BF16
def test_bf16_rounding_against_exact_rationals():
    rng = np.random.default_rng(11)
    x = rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000)
    # near-ties that a double->float->bf16 path would double-round
    base = rng.standard_normal(1000).astype(np.float32)
    b = np.frombuffer(base.tobytes(), dtype=np.uint32)
    tie = ((b & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32).astype(np.float64)
    x = np.concatenate([x, tie, tie * (1 + 2.0 ** -40), tie * (1 - 2.0 ** -40), [0.0, -0.0, 1.0, -3.0]])
    got = bits_to_f64(oracle.bf16_from_double(x))
    want = np.array([bf16_round_exact(Fraction(float(v))) for v in x])
    assert np.array_equal(got, want)


def test_bf16_rounding_matches_torch_on_floats():
    rng = np.random.default_rng(12)
    f = (rng.standard_normal(200000) * 10.0 ** rng.integers(-20, 20, 200000)).astype(np.float32)
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_from_double(f.astype(np.float64))
    assert np.array_equal(got, want)


# ----------------------------------------------------------------------- GEMM
@pytest.mark.parametrize("M,N,K,seed", [(1, 1, 128, 0), (7, 5, 256, 1), (130, 129, 384, 2),
                                        (200, 256, 256, 3), (33, 300, 128, 4),
                                        # K tails: one partial block, and full blocks + a partial one
                                        (5, 9, 16, 6), (40, 130, 200, 7), (129, 7, 272, 8)])
def test_gemm_ref_against_exact_brute_force(M, N, K, seed):
    rng = np.random.default_rng(seed)
    Kb = -(-K // 128)
    A = random_finite_codes(rng, (M, K))
    B = random_finite_codes(rng, (N, K))
    sA = random_scales(rng, (-(-M // 128), Kb))
    sB = random_scales(rng, (-(-N // 128), Kb))
    ref = oracle.gemm_ref(A, sA, B, sB)
    exact, absum = exact_ref(A, sA, B, sB, with_abs=True)
    ex = np.array([[float(v) for v in row] for row in exact])
    # FP64 error of a Kb-term sum of exactly-partialled terms: a few ulps of sum|term|
    assert np.all(np.abs(ref - ex) <= 2 * (Kb + 1) * 2.0 ** -53 * absum)
    # BF16 output: the oracle's rounding of its FP64 value against the exact rounding
    got = bits_to_f64(oracle.bf16_from_double(ref))
    want = np.array([[bf16_round_exact(v) for v in row] for row in exact])
    same = np.mean(got == want)
    assert same >= 0.9999
    ulp = np.abs(want) * 2.0 ** -7
    assert np.all(np.abs(got - want) <= ulp + 1e-300)


def test_gemm_ref_exact_small_integers():
    """Integer codes, power-of-two scales: the result is a dyadic value BF16 holds exactly."""
    rng = np.random.default_rng(5)
    M, N, K = 160, 136, 256
    tab = oracle.e4m3_table()
    code_of = {float(tab[c]): c for c in range(0x7F)}
    vals_a = rng.choice([-1, 0, 0, 0, 0, 0, 1], size=(M, K))
    vals_b = rng.choice([-2, -1, 0, 0, 0, 0, 0, 1, 2], size=(N, K))
    enc = lambda v: np.vectorize(lambda x: code_of[abs(float(x))] | (0x80 if x < 0 else 0))(v).astype(np.uint8)
    A, B = enc(vals_a), enc(vals_b)
    sA = (2.0 ** rng.integers(-1, 2, size=(2, 2))).astype(np.float32)
    sB = (2.0 ** rng.integers(-1, 1, size=(2, 2))).astype(np.float32)
    ref = oracle.gemm_ref(A, sA, B, sB)
    # exact value with integers: sum_kb s * P_kb
    want = np.zeros((M, N))
    for kb in range(2):
        sl = slice(128 * kb, 128 * kb + 128)
        P = vals_a[:, sl].astype(np.int64) @ vals_b[:, sl].astype(np.int64).T
        s = np.outer(sA[np.arange(M) // 128, kb], sB[np.arange(N) // 128, kb])
        want += s * P
    assert np.array_equal(ref, want)
    assert np.max(np.abs(want)) < 64 and np.all(np.mod(want * 4, 1) == 0)
    assert np.array_equal(bits_to_f64(oracle.bf16_from_double(ref)), want)


def test_gemm_ref_identity():
    rng = np.random.default_rng(6)
    M = K = 256
    N = 200
    A = np.zeros((M, K), dtype=np.uint8)
    A[np.arange(M), np.arange(M)] = 0x38          # E4M3 code of 1.0
    assert torch_decode(np.array([0x38]))[0] == 1.0
    sA = np.ones((2, 2), dtype=np.float32)
    B = random_finite_codes(rng, (N, K))
    sB = random_scales(rng, (2, 2))
    ref = oracle.gemm_ref(A, sA, B, sB)
    want = sB[np.arange(N)[None, :] // 128, np.arange(M)[:, None] // 128].astype(np.float64) * torch_decode(B).T
    assert np.array_equal(ref, want)


def test_gemm_ref_unit_scales_is_plain_dot():
    rng = np.random.default_rng(8)
    M, N, K = 64, 96, 512
    A = random_finite_codes(rng, (M, K), max_code=0x60)
    B = random_finite_codes(rng, (N, K), max_code=0x60)
    ones_a = np.ones((1, 4), np.float32)
    ones_b = np.ones((1, 4), np.float32)
    ref = oracle.gemm_ref(A, ones_a, B, ones_b)
    want = (codes_to_int(A) @ codes_to_int(B).T).astype(np.float64) / 2.0 ** 18
    assert np.array_equal(ref, want)


def test_gemm_ref_row_block_doubling_and_transpose():
    rng = np.random.default_rng(9)
    M, N, K = 300, 260, 384
    A = random_finite_codes(rng, (M, K))
    B = random_finite_codes(rng, (N, K))
    sA = random_scales(rng, (3, 3))
    sB = random_scales(rng, (3, 3))
    ref = oracle.gemm_ref(A, sA, B, sB)
    sA2 = sA.copy()
    sA2[1, :] *= 2
    ref2 = oracle.gemm_ref(A, sA2, B, sB)
    rows = np.arange(M)
    inside = (rows >= 128) & (rows < 256)
    assert np.array_equal(ref2[inside], 2 * ref[inside])
    assert np.array_equal(ref2[~inside], ref[~inside])
    # C^T = B.A^T with the roles of the operands swapped
    refT = oracle.gemm_ref(B, sB, A, sA)
    assert np.array_equal(refT, ref.T)


def test_gemm_ref_kblock_permutation():
    rng = np.random.default_rng(10)
    M, N, K = 130, 140, 512
    A = random_finite_codes(rng, (M, K))
    B = random_finite_codes(rng, (N, K))
    sA = random_scales(rng, (2, 4))
    sB = random_scales(rng, (2, 4))
    perm = np.array([2, 0, 3, 1])
    cols = (perm[:, None] * 128 + np.arange(128)[None, :]).reshape(-1)
    ref = oracle.gemm_ref(A, sA, B, sB)
    refp = oracle.gemm_ref(A[:, cols], sA[:, perm], B[:, cols], sB[:, perm])
    # only the FP64 summation order of the K-block terms changes
    exact, absum = exact_ref(A, sA, B, sB, with_abs=True)
    ex = np.array([[float(v) for v in row] for row in exact])
    bound = 2 * 5 * 2.0 ** -53 * absum
    assert np.all(np.abs(ref - ex) <= bound) and np.all(np.abs(refp - ex) <= bound)


def test_gemm_ref_row_and_col_subsets():
    rng = np.random.default_rng(13)
    M, N, K = 260, 270, 256
    A = random_finite_codes(rng, (M, K))
    B = random_finite_codes(rng, (N, K))
    sA = random_scales(rng, (3, 2))
    sB = random_scales(rng, (3, 2))
    full = oracle.gemm_ref(A, sA, B, sB)
    rows = np.array([0, 127, 128, 259])
    cols = np.array([269, 0, 130])
    sub = oracle.gemm_ref(A, sA, B, sB, rows=rows, cols=cols)
    assert np.array_equal(sub, full[np.ix_(rows, cols)])


def test_grouped_ref_equals_dense_per_expert():
    rng = np.random.default_rng(14)
    G, N, K = 4, 256, 256
    counts = np.array([130, 0, 5, 128])
    off = np.zeros(G + 1, np.int32)
    off[1:] = np.cumsum((counts + 127) // 128 * 128)
    Mt = int(off[-1])
    A = random_finite_codes(rng, (Mt + 128, K))       # one extra block owned by nobody
    sA = random_scales(rng, (Mt // 128 + 1, K // 128))
    B = random_finite_codes(rng, (G, N, K))
    sB = random_scales(rng, (G, N // 128, K // 128))
    rows = np.arange(Mt + 128)
    got = oracle.grouped_gemm_ref(A, sA, B, sB, off, rows)
    for g in range(G):
        r0, r1 = off[g], off[g + 1]
        if r0 == r1:
            continue
        dense = oracle.gemm_ref(A[r0:r1], sA[r0 // 128:r1 // 128], B[g], sB[g])
        assert np.array_equal(got[r0:r1], dense)
    assert np.all(np.isnan(got[Mt:]))


# ------------------------------------------------------------------- quantizer
def _quant_case(R, C, seed, outlier=False, zero_block=False):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((R, C), generator=g)
    if outlier:
        x[R // 3] *= 50.0
    if zero_block:
        x[:128, :128] = 0.0
        x[0, 0] = -0.0
    return x.to(torch.bfloat16)


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("R,C", [(1, 16), (128, 128), (200, 384), (257, 144), (64, 1040)])
def test_quantizer_roundtrip_bound_and_amax(R, C):
    x = _quant_case(R, C, R * 1000 + C, outlier=True)
    q, s = oracle.quantize_blockwise(_bits(x))
    xv = x.to(torch.float64).numpy()
    dec = oracle.e4m3_decode(q)
    tab = oracle.e4m3_table()[:0x7F]
    for br in range(s.shape[0]):
        for bc in range(s.shape[1]):
            blk = (slice(128 * br, 128 * br + 128), slice(128 * bc, 128 * bc + 128))
            xb, qb, db = xv[blk], q[blk], dec[blk]
            amax = np.max(np.abs(xb))
            sc = float(s[br, bc])
            assert sc == np.float32(np.float32(amax) / np.float32(448.0))
            # the amax element lands on +-448
            assert np.any((qb & 0x7F) == 0x7E)
            # round trip: within half an E4M3 spacing (plus the FP32 rounding of x/s)
            v = np.abs(xb) / sc
            idx = np.clip(np.searchsorted(tab, v), 1, 126)
            spacing = tab[idx] - tab[idx - 1]
            err = np.abs(db * sc - xb) / sc
            assert np.all(err <= 0.5 * spacing * (1 + 1e-6) + 1e-12)


def test_quantizer_matches_torch_division_and_cast():
    x = _quant_case(384, 512, 99, outlier=True, zero_block=True)
    q, s = oracle.quantize_blockwise(_bits(x))
    xf = x.to(torch.float32)
    R, C = xf.shape
    blocks = xf.reshape(R // 128, 128, C // 128, 128)
    amax = blocks.abs().amax(dim=(1, 3))
    scale = torch.where(amax == 0, torch.ones_like(amax), amax / torch.tensor(448.0))
    assert np.array_equal(s, scale.numpy())
    v = blocks / scale[:, None, :, None]
    want = v.reshape(R, C).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, want)
    # the all-zero block: scale 1, codes zero with the sign kept
    assert s[0, 0] == 1.0 and q[0, 0] == 0x80 and np.all(q[:128, :128].ravel()[1:] == 0)


@pytest.mark.parametrize("K", [16, 112, 144, 400])
def test_gemm_ref_k_tail_equals_zero_padded_full_blocks(K):
    """A partial last K block is the full block with zero codes in the missing columns.

    Zero codes add exact zeros to the block partial, so padding A and B with zero
    columns up to a multiple of 128 (same scales) must give the same FP64 values bit
    for bit; and the tail block's scale pair must act on the tail columns only."""
    rng = np.random.default_rng(K)
    M, N = 70, 150
    Kb = -(-K // 128)
    A = random_finite_codes(rng, (M, K))
    B = random_finite_codes(rng, (N, K))
    sA = random_scales(rng, (-(-M // 128), Kb))
    sB = random_scales(rng, (-(-N // 128), Kb))
    ref = oracle.gemm_ref(A, sA, B, sB)
    Kp = 128 * Kb
    Ap = np.zeros((M, Kp), np.uint8); Ap[:, :K] = A
    Bp = np.zeros((N, Kp), np.uint8); Bp[:, :K] = B
    assert np.array_equal(oracle.gemm_ref(Ap, sA, Bp, sB), ref)
    # doubling the tail block's A scales doubles exactly the tail's contribution
    sA2 = sA.copy(); sA2[:, Kb - 1] *= 2
    head = np.zeros_like(A); head[:, :128 * (Kb - 1)] = A[:, :128 * (Kb - 1)]
    tail = oracle.gemm_ref(A, sA2, B, sB) - oracle.gemm_ref(head, sA2, B, sB)
    tail1 = ref - oracle.gemm_ref(head, sA, B, sB)
    assert np.allclose(tail, 2 * tail1, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_masked_ref_equals_contiguous_ref_on_packed_rows():
    """The masked layout and the grouped-contiguous layout hold the same tokens: the
    masked formula must give the contiguous routine's values bit for bit (two routines
    with different expert lookups), NaN past each count, and clamp counts to M_max."""
    rng = np.random.default_rng(31)
    G, Mmax, N, K = 4, 200, 144, 256
    counts = np.array([0, 200, 77, 129])
    A = random_finite_codes(rng, (G, Mmax, K))
    sA = random_scales(rng, (G, 2, 2))
    B = random_finite_codes(rng, (G, N, K))
    sB = random_scales(rng, (G, 2, 2))
    got = oracle.masked_gemm_ref(A, sA, B, sB, counts)
    # packed contiguous layout: expert g's rows at a 128-aligned offset, same m-block scales
    padded = (counts + 127) // 128 * 128
    off = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    Ac = np.zeros((int(off[-1]), K), np.uint8)
    sAc = np.ones((int(off[-1]) // 128, 2), np.float32)
    for g in range(G):
        Ac[off[g]:off[g] + counts[g]] = A[g, :counts[g]]
        nb = padded[g] // 128
        sAc[off[g] // 128:off[g] // 128 + nb] = sA[g, :nb]
    rows = np.concatenate([np.arange(off[g], off[g] + counts[g]) for g in range(G)]).astype(np.int64)
    want = oracle.grouped_gemm_ref(Ac, sAc, B, sB, off, rows)
    got_rows = np.concatenate([got[g, :counts[g]] for g in range(G)])
    assert np.array_equal(got_rows, want)
    for g in range(G):
        assert np.all(np.isnan(got[g, counts[g]:]))
    # clamping: a count past M_max acts as M_max, a negative one as 0
    clamped = oracle.masked_gemm_ref(A, sA, B, sB, np.array([-5, 999, 77, 129]))
    assert np.array_equal(clamped[1], got[1]) and np.all(np.isnan(clamped[0]))


# ------------------------------------------------ per-row (1 x 128 group) A scales
@pytest.mark.parametrize("R,C", [(1, 16), (130, 384), (64, 1040)])
def test_group_quantizer_matches_torch_division_and_cast(R, C):
    """One scale per row and 128-column group: torch's FP32 amax / 448 and its FP32
    division + float8 cast (a library routine) give the same scales and codes."""
    x = _quant_case(R, C, 7000 + R + C, outlier=True)
    x[0, :16] = 0.0  # a partial group of zeros when C == 16
    q, s = oracle.quantize_groups(_bits(x))
    xf = x.to(torch.float32)
    Cb = -(-C // 128)
    xp = torch.zeros((R, Cb * 128))
    xp[:, :C] = xf
    g = xp.reshape(R, Cb, 128)
    amax = g.abs().amax(dim=2)
    scale = torch.where(amax == 0, torch.ones_like(amax), amax / torch.tensor(448.0))
    assert np.array_equal(s, scale.numpy())
    want = (g / scale[:, :, None]).reshape(R, Cb * 128)[:, :C].to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, want)
    # every non-zero group holds a code at +-448
    for r in range(R):
        for b in range(Cb):
            if amax[r, b] > 0:
                assert np.any((q[r, 128 * b:128 * b + 128] & 0x7F) == 0x7E)


@pytest.mark.parametrize("M,N,K,seed", [(7, 5, 256, 41), (130, 129, 272, 42), (33, 300, 128, 43)])
def test_rowscale_gemm_against_exact_brute_force(M, N, K, seed):
    rng = np.random.default_rng(seed)
    Kb = -(-K // 128)
    A = random_finite_codes(rng, (M, K))
    B = random_finite_codes(rng, (N, K))
    sA = random_scales(rng, (M, Kb))
    sB = random_scales(rng, (-(-N // 128), Kb))
    ref = oracle.gemm_ref_rowscale(A, sA, B, sB)
    exact, absum = exact_ref(A, sA, B, sB, with_abs=True, a_rows=1)
    ex = np.array([[float(v) for v in row] for row in exact])
    assert np.all(np.abs(ref - ex) <= 2 * (Kb + 1) * 2.0 ** -53 * absum)


def test_rowscale_gemm_equals_block_gemm_when_rows_share_scales():
    """Per-row scales that repeat the 128-row block's scale give the block form, bit for bit."""
    rng = np.random.default_rng(44)
    M, N, K = 300, 200, 384
    A = random_finite_codes(rng, (M, K))
    B = random_finite_codes(rng, (N, K))
    sA = random_scales(rng, (3, 3))
    sB = random_scales(rng, (2, 3))
    rows_scales = np.ascontiguousarray(sA[np.arange(M) // 128])
    assert np.array_equal(oracle.gemm_ref_rowscale(A, rows_scales, B, sB), oracle.gemm_ref(A, sA, B, sB))
    # and a row's own scale acts on that row alone
    sr = rows_scales.copy()
    sr[5] *= 4
    a = oracle.gemm_ref_rowscale(A, sr, B, sB)
    b = oracle.gemm_ref_rowscale(A, rows_scales, B, sB)
    assert np.array_equal(np.delete(a, 5, 0), np.delete(b, 5, 0))
    assert np.allclose(a[5], 4 * b[5], rtol=1e-15, atol=0)
