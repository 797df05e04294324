"""GPU parity of dg_quantize_blockwise: the E4M3 codes and the FP32 scales must be
bit-identical to the oracle quantizer on the same BF16 input."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_scales_b200 import binding, inputs

from parity import oracle_quant

pytestmark = pytest.mark.gpu


def run_and_compare(x: torch.Tensor):
    q_ref, s_ref = oracle_quant(x)
    q, s = binding.quantize_blockwise(x.cuda())
    torch.cuda.synchronize()
    q = q.cpu().numpy()
    s = s.cpu().numpy()
    assert s.shape == s_ref.shape
    assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32)), "scales differ"
    bad = np.flatnonzero(q.ravel() != q_ref.ravel())
    assert bad.size == 0, (bad.size, bad[:8], q.ravel()[bad[:8]], q_ref.ravel()[bad[:8]],
                           x.float().ravel()[bad[:8]].tolist())


@pytest.mark.parametrize("R,C", [(1, 16), (128, 128), (129, 144), (300, 1040), (512, 512), (77, 4096)])
def test_quantize_ragged_shapes(R, C):
    run_and_compare(inputs.bf16_normal((R, C), 1.0, 7000 + R + C))


def test_quantize_zero_blocks_and_signed_zeros():
    x = inputs.bf16_normal((256, 384), 1.0, 7100)
    x[:128, :128] = 0.0
    x[:128, :128].view(torch.int16)[::2, ::3] = -32768  # -0.0
    x[128:, 256:] = -0.0
    x[5, 300] = 0.0
    run_and_compare(x)
    q, s = binding.quantize_blockwise(x.cuda())
    assert s[0, 0].item() == 1.0 and s[1, 2].item() == 1.0


def test_quantize_rounding_boundaries():
    """Blocks whose scale is exactly a power of two put x/s on E4M3 midpoints,
    their FP32 neighbours, subnormal midpoints and the saturation edge."""
    tab = oracle.e4m3_table()[:0x7F]
    mids = (tab[:-1] + tab[1:]) / 2
    vals = np.concatenate([mids, tab, -mids, mids * (1 + 2.0 ** -7), mids * (1 - 2.0 ** -7)])
    vals = torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)
    n = vals.numel()
    x = torch.zeros((128, 1024), dtype=torch.bfloat16)
    flat = x.view(-1)
    reps = flat.numel() // n
    flat[:reps * n] = vals.repeat(reps)
    x[0, 0] = 448.0   # amax = 448 in every 128x128 block -> s = 1 exactly
    for b in range(8):
        x[0, 128 * b] = 448.0
    # a second copy scaled so s = 2^-4, and one with s = 2^5
    y = torch.cat([x, (x.float() * 2.0 ** -4).to(torch.bfloat16), (x.float() * 32).to(torch.bfloat16)], 0)
    run_and_compare(y)


def _bf16_from_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


def test_quantize_every_bf16_pattern_under_a_scale_sweep():
    """Every finite BF16 value, under block scales that are powers of two (x/s then
    lands exactly on E4M3 values, midpoints and their neighbours), one BF16 step above
    and below them, and a few arbitrary ones: the codes and scales must equal the
    oracle's (which divides in FP64 and rounds once) bit for bit.  Each 128x128 block
    holds the patterns not larger than its amax plus one element equal to it."""
    pos = np.arange(0x0000, 0x7F80, dtype=np.uint32)            # +0 .. largest finite
    bits = np.concatenate([pos, pos | 0x8000])                    # and their negatives
    mag = (pos.astype(np.uint32) << 16).view(np.float32)
    mag = np.concatenate([mag, mag])
    amaxes = []
    for k in (-40, -20, -10, -4, -1, 0, 1, 4, 12):
        a = np.array([448.0 * 2.0 ** k], np.float32)
        a_bits = int(torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).item()) & 0xFFFF
        amaxes += [a_bits, a_bits + 1, a_bits - 1]                # s a power of two, just above, just below
    for v in (1.0, 3.0, 0.1, 7.7e-3, 1234.5):
        amaxes.append(int(torch.tensor([v]).to(torch.bfloat16).view(torch.int16).item()) & 0xFFFF)
    blocks = []
    for a_bits in amaxes:
        a = float(np.array([a_bits << 16], np.uint32).view(np.float32)[0])
        sel = bits[mag <= a]
        per = 128 * 128 - 1
        for i in range(0, sel.size, per):
            blk = np.zeros(128 * 128, np.uint32)
            chunk = sel[i:i + per]
            blk[:chunk.size] = chunk
            blk[-1] = a_bits                                      # the block's amax
            blocks.append(blk.reshape(128, 128))
    x = _bf16_from_bits(np.concatenate(blocks, 0))
    assert x.shape[0] >= 128 * len(amaxes)
    run_and_compare(x)


def test_quantize_outlier_rows_4096():
    run_and_compare(inputs.dense_4096_outliers().A)


def test_quantize_wide_dynamic_range():
    g = torch.Generator().manual_seed(7200)
    x = torch.randn((384, 768), generator=g) * torch.exp(torch.randn((384, 768), generator=g) * 6)
    run_and_compare(x.to(torch.bfloat16))


@pytest.mark.slow
def test_quantize_full_moe_weights():
    """B of the 64-expert workload: 64 x 2048 x 7168 BF16, quantized as one
    [G*N][K] matrix (expert blocks never straddle since N % 128 == 0)."""
    w = inputs.moe_g64_zipf().B
    run_and_compare(w.reshape(-1, w.shape[-1]))


def test_quantize_determinism_and_noop():
    x = inputs.bf16_normal((300, 512), 1.0, 7300).cuda()
    q1, s1 = binding.quantize_blockwise(x)
    q2, s2 = binding.quantize_blockwise(x)
    assert torch.equal(q1, q2) and torch.equal(s1, s2)
    z = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    q, s = binding.quantize_blockwise(z)
    assert q.numel() == 0
