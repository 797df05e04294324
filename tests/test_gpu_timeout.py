"""Failure detection on the GPU without a fault: every pipeline wait in the kernels
is bounded.  A test hook makes a kernel's TMA producer skip its first stage,
so the MMA warp's wait for that stage can never succeed; the kernel must give up
after the (shortened) time limit, record DG_ERR_TIMEOUT in the device status word,
release its tensor memory and return, leaving the context usable."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_scales_b200 import binding, inputs

from parity import c_f64, check, dev, oracle_quant

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kernel", ["tile", "pair"])
def test_bounded_wait_reports_timeout_and_context_survives(kernel):
    d = inputs.dense_custom(256, 512, 512, seed=9500)
    qa, sa = oracle_quant(d.A)
    qb, sb = oracle_quant(d.B)
    A, SA, B, SB = dev(qa), dev(sa), dev(qb), dev(sb)
    assert binding.last_device_status() == 0
    try:
        binding.set_kernel_control(timeout_ns=50_000_000, debug_flags=1)
        binding.gemm_blockscaled(A, SA, B, SB, kernel=kernel)
        status = binding.last_device_status()
    finally:
        binding.set_kernel_control(0, 0)
    assert status == 6, f"expected DG_ERR_TIMEOUT, got {status}"
    # the same context still computes correct results
    c = c_f64(binding.gemm_blockscaled(A, SA, B, SB, kernel=kernel))
    assert binding.last_device_status() == 0
    check(c, oracle.gemm_ref(qa, sa, qb, sb), None, "after timeout")


@pytest.mark.parametrize("fused", [False, True])
def test_skinny_cluster_kernel_times_out_cleanly(fused):
    """The split-K skinny kernel gives up inside a thread-block cluster: every CTA of the
    cluster still reaches the cluster barriers, frees its tensor memory and returns."""
    M, N, K = 1 if fused else 16, 1024, 2048
    d = inputs.dense_custom(M, N, K, seed=9550)
    qa, sa = oracle_quant(d.A)
    qb, sb = oracle_quant(d.B)
    A, SA, B, SB = dev(qa), dev(sa), dev(qb), dev(sb)
    Abf = d.A.cuda()

    def call():
        if fused:
            return binding.gemm_blockscaled_bf16a(Abf, B, SB, kernel="fused")[0]
        return binding.gemm_blockscaled(A, SA, B, SB, kernel="skinny")

    assert binding.last_device_status() == 0
    try:
        binding.set_kernel_control(timeout_ns=50_000_000, debug_flags=1)
        call()
        status = binding.last_device_status()
    finally:
        binding.set_kernel_control(0, 0)
    assert status == 6, f"expected DG_ERR_TIMEOUT, got {status}"
    c = c_f64(call())
    assert binding.last_device_status() == 0
    check(c, oracle.gemm_ref(qa, sa, qb, sb), None, "after timeout")
