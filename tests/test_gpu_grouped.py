"""GPU parity of the MoE grouped-contiguous GEMM against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_scales_b200 import binding, inputs

from parity import c_f64, check, dev, grouped_ref_rows, oracle_quant, rows_per_quarter

pytestmark = pytest.mark.gpu


def quantized(w):
    qa, sa = oracle_quant(w.A)
    qb, sb = oracle_quant(w.B)
    return qa, sa, qb, sb


def run(qa, sa, qb, sb, off, capacity=None, fill=None):
    Mt, K = qa.shape
    cap = capacity or Mt
    A = torch.zeros((cap, K), dtype=torch.uint8, device="cuda")
    A[:Mt] = dev(qa)
    SA = torch.ones((cap // 128, -(-K // 128)), dtype=torch.float32, device="cuda")
    SA[:Mt // 128] = dev(sa)
    C = torch.full((cap, qb.shape[1]), fill if fill is not None else 0.0, dtype=torch.bfloat16, device="cuda")
    binding.grouped_gemm_contiguous(A, SA, dev(qb), dev(sb), dev(off), C=C)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    return C


@pytest.mark.parametrize("G,N,K,counts", [
    (4, 256, 256, [130, 0, 5, 128]),
    (3, 384, 640, [1, 300, 0]),
    (1, 128, 128, [77]),
    (6, 512, 384, [0, 0, 129, 64, 0, 256]),
    (2, 256, 208, [130, 60]),  # K tail: partial last K block
])
def test_grouped_small_full_compare(G, N, K, counts):
    w = inputs.grouped_custom(G, N, K, counts, seed=9000 + G + N)
    qa, sa, qb, sb = quantized(w)
    cap = w.M_total + 256  # rows past off[G] must stay untouched
    C = run(qa, sa, qb, sb, w.offsets, capacity=cap, fill=-3.0)
    c = c_f64(C)
    Mt = w.M_total
    rows = np.arange(Mt)
    ref = oracle.grouped_gemm_ref(qa, sa, qb, sb, w.offsets, rows)
    real = inputs.real_row_mask(w.counts, w.offsets)
    rms = float(np.sqrt(np.mean(ref[real] ** 2))) if real.any() else 0.0
    check(c[:Mt][real], ref[real], rms, "grouped real rows")
    assert np.all(c[:Mt][~real] == 0.0), "padding rows must come out zero"
    assert np.all(c[Mt:] == -3.0), "rows past off[G] were written"


def test_grouped_equals_dense_per_expert():
    w = inputs.grouped_custom(3, 512, 512, [200, 64, 390], seed=9100)
    qa, sa, qb, sb = quantized(w)
    C = run(qa, sa, qb, sb, w.offsets)
    for g in range(3):
        r0, r1 = int(w.offsets[g]), int(w.offsets[g + 1])
        d = binding.gemm_blockscaled(dev(qa[r0:r1]), dev(sa[r0 // 128:r1 // 128]), dev(qb[g]), dev(sb[g]),
                                     kernel="tile")
        torch.cuda.synchronize()
        assert torch.equal(d.view(torch.int16), C[r0:r1].view(torch.int16))


def test_grouped_offsets_read_on_device():
    """group_offsets produced on the device by an earlier kernel on the same stream."""
    counts = [128, 256, 0, 100]
    w = inputs.grouped_custom(4, 256, 256, counts, seed=9200)
    qa, sa, qb, sb = quantized(w)
    off_dev = torch.zeros(5, dtype=torch.int32, device="cuda")
    padded = torch.tensor([(c + 127) // 128 * 128 for c in counts], dtype=torch.int32, device="cuda")
    off_dev[1:] = torch.cumsum(padded, 0).to(torch.int32)
    C = torch.zeros((w.M_total, 256), dtype=torch.bfloat16, device="cuda")
    binding.grouped_gemm_contiguous(dev(qa), dev(sa), dev(qb), dev(sb), off_dev, C=C)
    torch.cuda.synchronize()
    ref = oracle.grouped_gemm_ref(qa, sa, qb, sb, w.offsets, np.arange(w.M_total))
    real = inputs.real_row_mask(w.counts, w.offsets)
    check(c_f64(C)[real], ref[real], float(np.sqrt(np.mean(ref[real] ** 2))), "device offsets")


def _grouped_workload_check(w, full=False, seed=0):
    """All real rows (full), or one real row in every 32-row quarter of every 128-row
    block that holds tokens plus each expert's first and last real row: every tile
    of the schedule is compared either way.  Padding rows must be exactly zero."""
    qa, sa, qb, sb = quantized(w)
    C = run(qa, sa, qb, sb, w.offsets)
    c = c_f64(C)
    real = inputs.real_row_mask(w.counts, w.offsets)
    if full:
        rows = np.flatnonzero(real)
    else:
        rng = np.random.default_rng(seed)
        rows = set()
        for g in range(w.G):
            n = int(w.counts[g])
            if not n:
                continue
            r0 = int(w.offsets[g])
            rows.update([r0, r0 + n - 1])
            for b in range(0, n, 128):
                rows.update(rows_per_quarter(r0 + b, n - b, rng))
        rows = np.array(sorted(rows), dtype=np.int64)
    ref = grouped_ref_rows(qa, sa, qb, sb, w.offsets, rows)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    check(c[rows], ref, rms, w.name)
    assert np.all(c[~real] == 0.0)


def test_moe_g8_workload():
    """Every real row of the 8-expert workload (16384 token slots x 4096 columns)."""
    _grouped_workload_check(inputs.moe_g8(), full=True)


@pytest.mark.slow
def test_moe_g64_zipf_workload():
    _grouped_workload_check(inputs.moe_g64_zipf())


@pytest.mark.parametrize("bad", ["not_a_multiple_of_128", "decreasing", "past_capacity", "nonzero_start"])
def test_grouped_malformed_offsets_leave_c_untouched_and_set_status(bad):
    """group_offsets that break their contract: the kernel computes nothing, records
    DG_ERR_GROUP_OFFSETS in the device status word (no trap, the context stays
    usable) and a correct call afterwards computes normally."""
    counts = [128, 256, 0, 100]
    w = inputs.grouped_custom(4, 256, 256, counts, seed=9300)
    qa, sa, qb, sb = quantized(w)
    off = w.offsets.copy()  # [0, 128, 384, 384, 512]
    cap = int(off[-1])
    if bad == "not_a_multiple_of_128":
        off[2] = 300
    elif bad == "decreasing":
        off[2] = 100
    elif bad == "past_capacity":
        off[4] = cap + 128
    else:
        off[0] = 128
    C = torch.full((cap, 256), -5.0, dtype=torch.bfloat16, device="cuda")
    binding.grouped_gemm_contiguous(dev(qa), dev(sa), dev(qb), dev(sb), dev(off), C=C)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 7
    assert torch.all(C == -5.0)
    assert binding.last_device_status() == 0  # the read cleared it
    C2 = run(qa, sa, qb, sb, w.offsets)
    ref = oracle.grouped_gemm_ref(qa, sa, qb, sb, w.offsets, np.arange(cap))
    real = inputs.real_row_mask(w.counts, w.offsets)
    check(c_f64(C2)[real], ref[real], float(np.sqrt(np.mean(ref[real] ** 2))), "after a malformed call")
