"""Host-side logic of bench.py that needs no GPU: the algorithmic work of each workload,
the whole-job aggregate, and the key of the ncu traffic figures."""
import importlib.util
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_code_hash_ignores_comments_only(bench):
    code = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    assert bench._code_only(code) == bench._code_only("/* doc */\n" + code.replace("// one more", "// edited"))
    assert bench._code_only(code) != bench._code_only(code.replace("+ 1", "+ 2"))
    # every traffic entry is keyed by the current code of its kernel file
    for (workload, fname, h), traffic in bench.NCU_TRAFFIC.items():
        assert bench.kernel_source_hash(fname) == h, (workload, fname)
        assert bench.ncu_traffic(workload, fname) == traffic
        # keyed by the file of the kernel the bench looks up for that workload
        assert fname == bench.kernel_file_of(workload), (workload, fname)
    assert bench.ncu_traffic("dense_512", "gemm_pair.cu") is None  # keyed by the dispatched kernel only
    assert bench.kernel_file_of("dense_8192") == "gemm_tile.cu"
    assert bench.kernel_file_of("moe_g64_zipf") == "gemm_tile.cu"
    assert bench.kernel_file_of("skinny_m1_fused") == "gemm_skinny.cu"


def test_dense_and_skinny_algorithmic_work(bench):
    from fp8_block_scaled_scales_b200 import inputs
    w = inputs.Dense("d", 4096, 4096, 4096, None, None, 0, np.zeros(0, np.int64))
    flops, nbytes, rows, cfg = bench.workload_facts(w)
    assert flops == 2.0 * 4096 ** 3 and rows == 4096
    # A + B codes, C in BF16, one FP32 scale per 128x128 block of A and of B
    assert nbytes == 4096 * 4096 * 2 + 4096 * 4096 * 2 + 4 * 32 * (32 + 32)
    assert cfg["M"] == cfg["N"] == cfg["K"] == 4096


def test_grouped_and_masked_count_real_tokens(bench):
    from fp8_block_scaled_scales_b200 import inputs
    counts = np.array([130, 0, 5])
    g = inputs.Grouped("g", 3, 256, 256, counts, inputs.padded_offsets(counts), None, None, 0)
    flops, nbytes, rows, _ = bench.workload_facts(g)
    assert flops == 2.0 * 135 * 256 * 256 and rows == 384  # 256 + 0 + 128 padded rows
    m = inputs.Masked("m", 3, 512, 256, 256, counts, None, None, 0)
    flops, nbytes, rows, cfg = bench.workload_facts(m)
    assert flops == 2.0 * 135 * 256 * 256 and rows == 3 * 512
    mblocks = 2 + 0 + 1  # m-blocks that hold tokens
    assert nbytes == mblocks * 128 * (256 + 2 * 256) + 3 * 256 * 256 + 4 * (mblocks + 3 * 2) * 2
    assert cfg["m_max"] == 512


def test_whole_job_rate_is_replicas_over_slowest(bench):
    assert bench.aggregate_rate(1, 1e12, 1.0) == pytest.approx(1e15)
    assert bench.aggregate_rate(8, 1e12, 2.0) == pytest.approx(8e12 / 2e-3)


def test_e2e_copies_a_masked_slabs_tokens_only(bench):
    from fp8_block_scaled_scales_b200 import inputs
    m = inputs.Masked("m", 3, 512, 256, 256, np.array([130, 0, 512]), None, None, 0)
    assert bench.io_rows(m, 3 * 512) == [(0, 130), (1024, 512)]
    d = inputs.Dense("d", 300, 256, 256, None, None, 0, np.zeros(0, np.int64))
    assert bench.io_rows(d, 300) == [(0, 300)]
