"""Seeded synthetic inputs for the FP8 block-scaled GEMM workloads.

This module holds random draws only: shapes, value distributions and MoE routing
structure.  It does no quantisation and no GEMM arithmetic, so the CUDA path and
the CPU oracle can both be fed from it without sharing any of the method.

Recipe (every draw is CPU-side and seeded, so any machine reproduces it):
  * BF16 matrices: FP32 standard normal from torch.Generator(seed), times std,
    rounded to BF16 (round to nearest even, torch's cast).
  * Outlier rows: a seeded sample without replacement of round(frac * rows)
    rows, multiplied by the factor in FP32 before the BF16 rounding.
  * MoE counts: a seeded numpy Generator draws expert probabilities (Dirichlet
    with all alphas 1, or p_i proportional to i^-s with the expert ids randomly
    permuted) and then the per-expert token-slot counts from a multinomial.
  * Grouped layout: each expert's rows padded up to a multiple of 128; padding
    rows of A are zero; group_offsets is the int32 prefix sum of padded counts.
  * Masked layout: expert g's tokens are rows 0..count_g-1 of its M_max-row slab;
    the rows after them hold N(0, 100^2) junk, which no output may depend on.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

ALIGN_M = 128


def bf16_normal(shape, std: float, seed: int) -> torch.Tensor:
    """CPU BF16 tensor of N(0, std^2) draws."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def moe_counts(G: int, slots: int, seed: int, dist: str = "dirichlet",
               zipf_s: float = 1.1) -> np.ndarray:
    """Per-expert token-slot counts (int64 [G]) summing to `slots`."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if dist == "dirichlet":
        p = rng.dirichlet(np.ones(G))
    elif dist == "zipf":
        w = np.arange(1, G + 1, dtype=np.float64) ** (-zipf_s)
        p = (w / w.sum())[rng.permutation(G)]
    else:
        raise ValueError(dist)
    return rng.multinomial(slots, p).astype(np.int64)


def padded_offsets(counts: np.ndarray, align: int = ALIGN_M) -> np.ndarray:
    """int32 [G+1] prefix sum of the counts, each rounded up to `align`."""
    padded = (np.asarray(counts, dtype=np.int64) + align - 1) // align * align
    off = np.zeros(len(counts) + 1, dtype=np.int64)
    np.cumsum(padded, out=off[1:])
    assert off[-1] < 2**31
    return off.astype(np.int32)


def real_row_mask(counts: np.ndarray, offsets: np.ndarray) -> np.ndarray:
    """bool [offsets[-1]]: True for rows that hold a routed token (not padding)."""
    mask = np.zeros(int(offsets[-1]), dtype=bool)
    for g, c in enumerate(counts):
        mask[offsets[g]:offsets[g] + c] = True
    return mask


@dataclass
class Dense:
    name: str
    M: int
    N: int
    K: int
    A: torch.Tensor          # bf16 [M][K]
    B: torch.Tensor          # bf16 [N][K]
    seed: int
    outliers: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))


@dataclass
class Grouped:
    name: str
    G: int
    N: int
    K: int
    counts: np.ndarray       # int64 [G] real token slots per expert
    offsets: np.ndarray      # int32 [G+1] padded prefix sum
    A: torch.Tensor          # bf16 [offsets[-1]][K], padding rows zero
    B: torch.Tensor          # bf16 [G][N][K]
    seed: int

    @property
    def M_total(self) -> int:
        return int(self.offsets[-1])


def _dense(name, M, N, K, seed, std_a, std_b, outlier_frac=0.0):
    ga = torch.Generator().manual_seed(seed)
    a = torch.randn((M, K), generator=ga, dtype=torch.float32)
    if std_a != 1.0:
        a.mul_(std_a)
    outl = np.zeros(0, np.int64)
    if outlier_frac > 0.0:
        n_out = int(round(outlier_frac * M))
        idx = torch.randperm(M, generator=ga)[:n_out]
        a[idx] *= 50.0
        outl = np.sort(idx.numpy().astype(np.int64))
    b = bf16_normal((N, K), std_b, seed + 500_000)
    return Dense(name, M, N, K, a.to(torch.bfloat16), b, seed, outl)


def _grouped(name, G, N, K, slots, seed, dist):
    counts = moe_counts(G, slots, seed, dist)
    off = padded_offsets(counts)
    Mt = int(off[-1])
    ga = torch.Generator().manual_seed(seed)
    a = torch.zeros((Mt, K), dtype=torch.bfloat16)
    real = int(counts.sum())
    draws = torch.randn((real, K), generator=ga, dtype=torch.float32).to(torch.bfloat16)
    pos = 0
    for g in range(G):
        c = int(counts[g])
        a[off[g]:off[g] + c] = draws[pos:pos + c]
        pos += c
    b = bf16_normal((G, N, K), 0.02, seed + 500_000)
    return Grouped(name, G, N, K, counts, off, a, b, seed)


# The workloads (seed 1000 + workload number; the masked MoE layout is number 7).
def dense_512() -> Dense:
    """M=N=K=512, A and B from N(0,1)."""
    return _dense("dense_512", 512, 512, 512, 1001, 1.0, 1.0)


def dense_4096_outliers() -> Dense:
    """M=N=K=4096, A from N(0,1) with 1% of rows x50, B from N(0,0.02)."""
    return _dense("dense_4096_outliers", 4096, 4096, 4096, 1002, 1.0, 0.02, outlier_frac=0.01)


def skinny(M: int) -> Dense:
    """M in {1,16,64,128}, N=K=4096, A from N(0,1), B from N(0,0.02)."""
    return _dense(f"skinny_m{M}", M, 4096, 4096, 1003, 1.0, 0.02)


def moe_g8() -> Grouped:
    """8 experts, N=K=4096, 8192 tokens x top-2 slots, Dirichlet(1) routing."""
    return _grouped("moe_g8_n4096_k4096", 8, 4096, 4096, 16384, 1004, "dirichlet")


def moe_g64_zipf() -> Grouped:
    """64 experts, N=2048, K=7168, 32768 slots, Zipf(1.1)-skewed routing."""
    return _grouped("moe_g64_n2048_k7168", 64, 2048, 7168, 32768, 1005, "zipf")


def dense_8192() -> Dense:
    """M=N=K=8192, A from N(0,1), B from N(0,0.02)."""
    return _dense("dense_8192", 8192, 8192, 8192, 1006, 1.0, 0.02)


def dense_custom(M: int, N: int, K: int, seed: int, std_a=1.0, std_b=0.02,
                 outlier_frac=0.0) -> Dense:
    return _dense(f"dense_{M}x{N}x{K}", M, N, K, seed, std_a, std_b, outlier_frac)


def grouped_custom(G: int, N: int, K: int, counts, seed: int) -> Grouped:
    """Grouped layout with the given per-expert counts (zeros allowed)."""
    counts = np.asarray(counts, dtype=np.int64)
    off = padded_offsets(counts)
    Mt = int(off[-1])
    ga = torch.Generator().manual_seed(seed)
    a = torch.zeros((Mt, K), dtype=torch.bfloat16)
    for g in range(G):
        c = int(counts[g])
        if c:
            a[off[g]:off[g] + c] = torch.randn((c, K), generator=ga).to(torch.bfloat16)
    b = bf16_normal((G, N, K), 0.02, seed + 500_000)
    return Grouped(f"grouped_g{G}_n{N}_k{K}", G, N, K, counts, off, a, b, seed)


@dataclass
class Masked:
    name: str
    G: int
    M_max: int
    N: int
    K: int
    counts: np.ndarray   # int64 [G], tokens per expert
    A: torch.Tensor      # BF16 [G][M_max][K]; rows >= counts[g] are junk
    B: torch.Tensor      # BF16 [G][N][K]
    seed: int


def masked_custom(G: int, M_max: int, N: int, K: int, counts, seed: int) -> Masked:
    """Masked MoE layout with the given per-expert counts (0..M_max)."""
    counts = np.asarray(counts, dtype=np.int64)
    ga = torch.Generator().manual_seed(seed)
    a = torch.randn((G, M_max, K), generator=ga, dtype=torch.float32)
    for g in range(G):
        a[g, int(counts[g]):] *= 100.0
    b = bf16_normal((G, N, K), 0.02, seed + 500_000)
    return Masked(f"masked_g{G}_m{M_max}_n{N}_k{K}", G, M_max, N, K, counts, a.to(torch.bfloat16), b, seed)


def moe_masked_g8() -> Masked:
    """The moe_g8 routing (8 experts, N=K=4096, 16384 slots, Dirichlet(1)) in the
    masked layout: slabs of M_max = the largest count rounded up to 128."""
    counts = moe_counts(8, 16384, 1004, "dirichlet")
    m_max = int((counts.max() + ALIGN_M - 1) // ALIGN_M * ALIGN_M)
    m = masked_custom(8, m_max, 4096, 4096, counts, 1007)
    m.name = "moe_masked_g8_n4096_k4096"
    return m


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 view of a CPU BF16 tensor (no copy of the values' meaning)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
