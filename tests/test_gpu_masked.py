"""GPU parity of the masked MoE GEMM (per-expert token counts read on the device)."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_scales_b200 import binding, inputs

from parity import c_f64, check, dev, oracle_quant, oracle_quant_tokens

pytestmark = pytest.mark.gpu


def quantized(w, junk_seed=None):
    qa, sa = oracle_quant_tokens(w.A, w.counts)  # [G][M_max][K], [G][ceil(M_max/128)][Kb]
    qb, sb = oracle_quant(w.B)
    if junk_seed is not None:
        # rows past each count may hold anything, NaN codes included: no output may see them
        rng = np.random.default_rng(junk_seed)
        for g in range(w.G):
            c = int(w.counts[g])
            qa[g, c:] = rng.integers(0, 256, size=qa[g, c:].shape, dtype=np.uint8)
    return qa, sa, qb, sb


def run(qa, sa, qb, sb, counts, fill=-3.0):
    G, Mmax, K = qa.shape
    N = qb.shape[1]
    C = torch.full((G, Mmax, N), fill, dtype=torch.bfloat16, device="cuda")
    mm = torch.from_numpy(np.asarray(counts, dtype=np.int32)).cuda()
    binding.grouped_gemm_masked(dev(qa), dev(sa), dev(qb), dev(sb), mm, C=C)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    return C


@pytest.mark.parametrize("G,Mmax,N,K,counts", [
    (4, 200, 256, 256, [0, 200, 77, 129]),
    (4, 256, 128, 4000, [256, 0, 1, 128]),      # narrow N (128-column tiles), K tail
    (3, 130, 384, 640, [130, 2, 65]),
    (1, 1000, 512, 384, [999]),
])
def test_masked_small_full_compare(G, Mmax, N, K, counts):
    w = inputs.masked_custom(G, Mmax, N, K, counts, seed=9500 + G + Mmax + N)
    qa, sa, qb, sb = quantized(w, junk_seed=9600 + G)
    C = c_f64(run(qa, sa, qb, sb, counts))
    ref = oracle.masked_gemm_ref(qa, sa, qb, sb, counts)
    real = np.concatenate([ref[g, :counts[g]] for g in range(G)])
    got = np.concatenate([C[g, :counts[g]] for g in range(G)])
    rms = float(np.sqrt(np.mean(real ** 2)))
    check(got, real, rms, "masked real rows")
    for g in range(G):
        assert np.all(C[g, counts[g]:] == -3.0), f"expert {g}: rows past its count were written"


def test_masked_counts_clamped_and_written_on_device():
    """Counts come from an earlier kernel on the stream; out-of-range ones are clamped."""
    G, Mmax, N, K = 3, 256, 256, 256
    counts = [300, -4, 100]  # clamped to 256, 0, 100
    w = inputs.masked_custom(G, Mmax, N, K, [256, 0, 100], seed=9700)
    qa, sa, qb, sb = quantized(w)
    mm = torch.tensor([0, 0, 0], dtype=torch.int32, device="cuda")
    mm += torch.tensor(counts, dtype=torch.int32, device="cuda")  # stream-ordered device write
    C = torch.full((G, Mmax, N), -3.0, dtype=torch.bfloat16, device="cuda")
    binding.grouped_gemm_masked(dev(qa), dev(sa), dev(qb), dev(sb), mm, C=C)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    ref = oracle.masked_gemm_ref(qa, sa, qb, sb, np.array(counts))
    c = c_f64(C)
    check(c[0], ref[0], None, "expert 0 (count clamped to M_max)")
    assert np.all(c[1] == -3.0)
    check(c[2, :100], ref[2, :100], None, "expert 2")
    assert np.all(c[2, 100:] == -3.0)


def test_masked_equals_contiguous_kernel_bitwise():
    """Same tokens in the contiguous layout: the same tile arithmetic, so the same bits."""
    G, Mmax, N, K = 3, 384, 512, 512
    counts = np.array([384, 130, 7])
    w = inputs.masked_custom(G, Mmax, N, K, counts, seed=9800)
    qa, sa, qb, sb = quantized(w)
    Cm = run(qa, sa, qb, sb, counts)
    padded = (counts + 127) // 128 * 128
    off = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    Ac = np.zeros((int(off[-1]), K), np.uint8)
    sAc = np.ones((int(off[-1]) // 128, K // 128), np.float32)
    for g in range(G):
        Ac[off[g]:off[g] + counts[g]] = qa[g, :counts[g]]
        sAc[off[g] // 128:off[g] // 128 + padded[g] // 128] = sa[g, :padded[g] // 128]
    Cc = binding.grouped_gemm_contiguous(dev(Ac), dev(sAc), dev(qb), dev(sb), dev(off))
    torch.cuda.synchronize()
    for g in range(G):
        a = Cm[g, :counts[g]].view(torch.int16)
        b = Cc[off[g]:off[g] + counts[g]].view(torch.int16)
        assert torch.equal(a, b), f"expert {g}"


def test_moe_masked_g8_workload_sampled():
    w = inputs.moe_masked_g8()
    qa, sa, qb, sb = quantized(w, junk_seed=9900)
    C = c_f64(run(qa, sa, qb, sb, w.counts))
    rng = np.random.default_rng(0)
    for g in range(w.G):
        c = int(w.counts[g])
        if c == 0:
            continue
        rows = np.unique(np.concatenate([[0, c - 1], rng.integers(0, c, 6)])).astype(np.int64)
        ref = oracle.gemm_ref(qa[g], sa[g], qb[g], sb[g], rows=rows)
        check(C[g][rows], ref, None, f"moe_masked_g8 expert {g}")
        assert np.all(C[g, c:] == -3.0)


def test_masked_largest_expert_count():
    """G = 256, the most the prefix table holds: many empty and one-token experts."""
    G, Mmax, N, K = 256, 128, 128, 128
    rng = np.random.default_rng(9950)
    counts = rng.choice([0, 0, 1, 7, 128, 64], size=G)
    w = inputs.masked_custom(G, Mmax, N, K, counts, seed=9951)
    qa, sa, qb, sb = quantized(w, junk_seed=9952)
    C = c_f64(run(qa, sa, qb, sb, counts))
    ref = oracle.masked_gemm_ref(qa, sa, qb, sb, counts)
    real = np.concatenate([ref[g, :counts[g]] for g in range(G) if counts[g]])
    got = np.concatenate([C[g, :counts[g]] for g in range(G) if counts[g]])
    check(got, real, float(np.sqrt(np.mean(real ** 2))), "masked G=256")
    for g in range(G):
        assert np.all(C[g, counts[g]:] == -3.0)


@pytest.mark.parametrize("G,Mmax,K,counts", [
    (4, 200, 256, [0, 200, 77, 129]),        # an empty slab, a full one, partial last blocks
    (3, 384, 4000, [384, 1, 128]),           # K tail; a block boundary exactly at the count
    (2, 130, 144, [-5, 1000]),               # counts clamped to [0, M_max]
    (2, 5120, 256, [5000, 2100]),            # 40 row blocks: each CTA of a slab takes several in turn
])
def test_masked_quantizer_quantizes_each_slabs_tokens_alone(G, Mmax, K, counts):
    """Slab g's first counts[g] rows get, bit for bit, the block quantizer's codes and
    scales for the matrix of those rows alone (its last block's amax covers tokens
    only); rows past the count and blocks past the last token keep what the buffers held."""
    clamped = np.clip(counts, 0, Mmax)
    w = inputs.masked_custom(G, Mmax, 128, K, clamped, seed=9300 + G + K)
    qa_ref, sa_ref = oracle_quant_tokens(w.A, clamped)
    mm = torch.from_numpy(np.asarray(counts, dtype=np.int32)).cuda()
    Q = torch.full((G, Mmax, K), 0xA5, dtype=torch.uint8, device="cuda")
    S = torch.full((G, (Mmax + 127) // 128, (K + 127) // 128), -7.0, dtype=torch.float32, device="cuda")
    binding.quantize_blockwise_masked(w.A.cuda(), mm, q=Q, s=S)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    Qh, Sh = Q.cpu().numpy(), S.cpu().numpy()
    for g in range(G):
        c = int(clamped[g])
        nb = (c + 127) // 128                    # blocks holding a token
        assert np.array_equal(Qh[g, :c], qa_ref[g, :c]), f"slab {g}: codes"
        assert np.array_equal(Sh[g, :nb].view(np.uint32), sa_ref[g, :nb].view(np.uint32)), f"slab {g}: scales"
        assert np.all(Qh[g, c:] == 0xA5) and np.all(Sh[g, nb:] == -7.0), f"slab {g}: rows past the count written"


def test_masked_quantizer_ignores_rows_past_the_count():
    """Changing the rows past each count (to anything, infinities and NaN included)
    changes no code or scale the quantizer writes."""
    G, Mmax, K, counts = 3, 256, 384, [77, 128, 200]
    w = inputs.masked_custom(G, Mmax, 128, K, counts, seed=9350)
    mm = torch.tensor(counts, dtype=torch.int32, device="cuda")
    A = w.A.cuda()
    q1, s1 = binding.quantize_blockwise_masked(A, mm)
    A2 = A.clone()
    rng = np.random.default_rng(9351)
    for g in range(G):
        junk = rng.integers(0, 1 << 16, size=(Mmax - counts[g], K), dtype=np.uint16)
        A2[g, counts[g]:] = torch.from_numpy(junk.view(np.int16)).cuda().view(torch.bfloat16)
    q2, s2 = binding.quantize_blockwise_masked(A2, mm)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert torch.equal(q1, q2) and torch.equal(s1.view(torch.int32), s2.view(torch.int32))


def test_masked_quantizer_feeds_the_masked_gemm_like_per_expert_quantization():
    """The masked GEMM on the masked quantizer's output equals, bit for bit, the masked
    GEMM on each expert's tokens quantized by the plain quantizer as a matrix of their own."""
    G, Mmax, N, K, counts = 4, 512, 256, 512, [300, 0, 129, 512]
    w = inputs.masked_custom(G, Mmax, N, K, counts, seed=9400)
    qb, sb = oracle_quant(w.B)
    mm = torch.from_numpy(np.asarray(counts, dtype=np.int32)).cuda()
    A = w.A.cuda()
    qa1, sa1 = binding.quantize_blockwise_masked(A, mm)
    qa2 = torch.zeros_like(qa1)
    sa2 = torch.ones_like(sa1)
    for g in range(G):
        if counts[g]:
            q, s = binding.quantize_blockwise(A[g, :counts[g]])
            qa2[g, :counts[g]] = q
            sa2[g, :s.shape[0]] = s
    C1 = binding.grouped_gemm_masked(qa1, sa1, dev(qb), dev(sb), mm)
    C2 = binding.grouped_gemm_masked(qa2, sa2, dev(qb), dev(sb), mm)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    for g in range(G):
        assert torch.equal(C1[g, :counts[g]].view(torch.int16), C2[g, :counts[g]].view(torch.int16))
