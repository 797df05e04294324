"""GPU parity of the GEMM that takes BF16 activations and quantizes them itself.

Both forms -- the block quantizer followed by the FP8 GEMM (the default), and for
M <= 16 the one-launch skinny kernel whose extra warps quantize A straight into
the MMA's stages -- must give the block quantizer's codes and scales bit for bit,
the same C, bit for bit, as the FP8 GEMM run on those codes (same kernel family,
same promotion order), and C within tolerance of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_scales_b200 import binding, inputs

from parity import c_f64, check, dev, oracle_quant

pytestmark = pytest.mark.gpu

SHAPES = [(1, 4096, 4096), (1, 272, 144), (1, 4096, 4000), (16, 4096, 4096), (17, 512, 640), (64, 1040, 768), (100, 256, 256),
          (128, 4096, 512), (33, 128, 4096), (5, 272, 144), (48, 384, 4000), (300, 512, 1152)]


CASES = [(M, N, K, "auto") for M, N, K in SHAPES] + [(M, N, K, "fused") for M, N, K in SHAPES if M <= 16]


@pytest.mark.parametrize("M,N,K,kernel", CASES)
def test_bf16a_gemm_matches_quantizer_and_fp8_gemm(M, N, K, kernel):
    d = inputs.dense_custom(M, N, K, seed=8700 + M + N + K)
    qa_ref, sa_ref = oracle_quant(d.A)
    qb, sb = oracle_quant(d.B)
    A = d.A.cuda()
    B, SB = dev(qb), dev(sb)
    C, QA, SA = binding.gemm_blockscaled_bf16a(A, B, SB, kernel=kernel)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    # the activations' codes and scales are exactly the block quantizer's
    assert np.array_equal(QA.cpu().numpy(), qa_ref), "codes differ from the block quantizer"
    assert np.array_equal(SA.cpu().numpy().view(np.uint32), sa_ref.view(np.uint32)), "scales differ"
    # C equals the FP8 GEMM on those codes, bit for bit
    C2 = binding.gemm_blockscaled(dev(qa_ref), dev(sa_ref), B, SB, kernel="auto")
    torch.cuda.synchronize()
    assert torch.equal(C.view(torch.int16), C2.view(torch.int16)), "fused and unfused results differ"
    check(c_f64(C), oracle.gemm_ref(qa_ref, sa_ref, qb, sb), None, f"bf16a {kernel} {M}x{N}x{K}")


@pytest.mark.parametrize("M,kernel", [(20, "auto"), (13, "fused")])
def test_bf16a_gemm_outputs_only_where_owned(M, kernel):
    """The codes/scales outputs are written exactly over [M][K] and [ceil(M/128)][Kb]."""
    N, K = 256, 400
    d = inputs.dense_custom(M, N, K, seed=8800)
    qb, sb = oracle_quant(d.B)
    guard = 4096
    qbuf = torch.full((M * K + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((4 + 2 * 64,), -5.0, dtype=torch.float32, device="cuda")
    QA = qbuf[guard:guard + M * K].view(M, K)
    SA = sbuf[64:64 + 4].view(1, 4)
    binding.gemm_blockscaled_bf16a(d.A.cuda(), dev(qb), dev(sb), QA=QA, sA=SA, kernel=kernel)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert torch.all(qbuf[:guard] == 0xA5) and torch.all(qbuf[guard + M * K:] == 0xA5)
    assert torch.all(sbuf[:64] == -5.0) and torch.all(sbuf[68:] == -5.0)
    qa_ref, sa_ref = oracle_quant(d.A)
    assert np.array_equal(QA.cpu().numpy(), qa_ref)
    assert np.array_equal(SA.cpu().numpy(), sa_ref)


@pytest.mark.parametrize("M,kernel", [(64, "auto"), (16, "fused"), (1, "fused")])
def test_bf16a_gemm_deterministic(M, kernel):
    N, K = 4096, 4096
    d = inputs.skinny(M)
    qb, sb = oracle_quant(d.B)
    A, B, SB = d.A.cuda(), dev(qb), dev(sb)
    outs = [binding.gemm_blockscaled_bf16a(A, B, SB, kernel=kernel)[0] for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(outs[0].view(torch.int16), o.view(torch.int16)) for o in outs[1:])


@pytest.mark.parametrize("M,kernel", [(64, "skinny"), (200, "tile"), (200, "pair"), (16, "fused")])
def test_bf16a_gemm_each_kernel_choice(M, kernel):
    """Every kernel the BF16-activation call can be asked for gives the quantizer's codes
    and scales bit for bit and C equal, bit for bit, to the FP8 GEMM of the same kernel
    on those codes."""
    N, K = 384, 640
    d = inputs.dense_custom(M, N, K, seed=8900 + M)
    qa_ref, sa_ref = oracle_quant(d.A)
    qb, sb = oracle_quant(d.B)
    B, SB = dev(qb), dev(sb)
    C, QA, SA = binding.gemm_blockscaled_bf16a(d.A.cuda(), B, SB, kernel=kernel)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert np.array_equal(QA.cpu().numpy(), qa_ref)
    assert np.array_equal(SA.cpu().numpy().view(np.uint32), sa_ref.view(np.uint32))
    C2 = binding.gemm_blockscaled(dev(qa_ref), dev(sa_ref), B, SB, kernel="skinny" if kernel == "fused" else kernel)
    torch.cuda.synchronize()
    assert torch.equal(C.view(torch.int16), C2.view(torch.int16))
    check(c_f64(C), oracle.gemm_ref(qa_ref, sa_ref, qb, sb), None, f"bf16a {kernel} {M}x{N}x{K}")


def test_bf16a_gemm_rejects_bad_kernel_choices():
    A = torch.zeros((17, 128), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((128, 128), dtype=torch.uint8, device="cuda")
    SB = torch.ones((1, 1), dtype=torch.float32, device="cuda")
    with pytest.raises(binding.DGError) as e:  # the one-launch form stops at 16 rows
        binding.gemm_blockscaled_bf16a(A, B, SB, kernel="fused")
    assert e.value.status == 2
    with pytest.raises(binding.DGError) as e:  # the FP8-input GEMM has no fused form
        binding.gemm_blockscaled(A.view(torch.uint8)[:, :128].contiguous(), torch.ones((1, 1), device="cuda"),
                                 B, SB, kernel="fused")
    assert e.value.status == 1
