"""Shared helpers for the GPU parity tests: run the oracle on the same seeded
inputs the CUDA path gets and compare element by element."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from fp8_block_scaled_scales_b200 import inputs


def oracle_quant(x_bf16: torch.Tensor):
    """Oracle quantization of a CPU BF16 tensor (2-D or 3-D, blocks per last two dims)."""
    if x_bf16.dim() == 3:
        qs, ss = zip(*(oracle.quantize_blockwise(inputs.bf16_bits(x_bf16[g])) for g in range(x_bf16.shape[0])))
        return np.stack(qs), np.stack(ss)
    return oracle.quantize_blockwise(inputs.bf16_bits(x_bf16))


def oracle_quant_tokens(x_bf16: torch.Tensor, counts):
    """Oracle quantization of masked-MoE activations [G][M_max][K]: the first counts[g]
    rows of slab g quantized as a matrix of their own.  Codes of the rows past a count
    are 0 and the scales of the blocks past the last token 1 (no output reads them)."""
    G, M_max, K = x_bf16.shape
    qa = np.zeros((G, M_max, K), np.uint8)
    sa = np.ones((G, -(-M_max // 128), -(-K // 128)), np.float32)
    for g in range(G):
        c = min(max(int(counts[g]), 0), M_max)
        if c:
            q, s = oracle.quantize_blockwise(inputs.bf16_bits(x_bf16[g, :c]))
            qa[g, :c], sa[g, :s.shape[0]] = q, s
    return qa, sa


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def c_f64(c: torch.Tensor) -> np.ndarray:
    return c.float().cpu().numpy().astype(np.float64)


def check(c_rows: np.ndarray, ref: np.ndarray, rms: float, what: str):
    ok, nbad, ratio = oracle.check_tolerance(c_rows, ref, rms)
    assert ok, f"{what}: {nbad} of {ref.size} outside |c-ref| <= 1e-2|ref| + 1e-3 rms (worst ratio {ratio:.3g})"
    return ratio


def stratified_rms(ref_rows: np.ndarray, row_weights: np.ndarray) -> float:
    """RMS over all rows of a matrix from a weighted sample of its rows."""
    ms = np.mean(ref_rows * ref_rows, axis=1)
    return float(np.sqrt(np.sum(ms * row_weights) / np.sum(row_weights)))


def grouped_ref_rows(qa, sa, qb, sb, offsets, rows):
    """Oracle values of the grouped-contiguous layout at `rows` (all columns), one
    dense oracle call per expert on the expert's slice: the grouped form is the dense
    formula per expert (pinned in the oracle tests), and the dense routine decodes
    each expert's weights once instead of once per row."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.full((rows.size, qb.shape[1]), np.nan)
    owner = np.searchsorted(offsets, rows, side="right") - 1
    for g in np.unique(owner):
        sel = np.flatnonzero(owner == g)
        r0, r1 = int(offsets[g]), int(offsets[g + 1])
        out[sel] = oracle.gemm_ref(qa[r0:r1], sa[r0 // 128:r1 // 128], qb[g], sb[g], rows=rows[sel] - r0)
    return out


def rows_per_quarter(first: int, count: int, rng) -> list:
    """One random row in each 32-row quarter of the 128-row block at `first` that
    holds any of the block's first `count` rows: every epilogue warp's output of
    every tile of that block is then checked."""
    rows = []
    for q0 in range(0, min(count, 128), 32):
        rows.append(first + q0 + int(rng.integers(0, min(32, count - q0))))
    return rows
