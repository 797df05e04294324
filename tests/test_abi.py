"""The C ABI: libdg.so builds, loads without a GPU, exports every symbol that
include/dg.h declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

from fp8_block_scaled_scales_b200 import binding
from fp8_block_scaled_scales_b200 import build as dgbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "dg.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    dgbuild.build()
    return binding.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("dg_quantize_blockwise", "dg_fp8_gemm_blockscaled", "dg_fp8_grouped_gemm_contiguous"):
        assert f in names
    assert set(names) == set(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_status_strings_and_version(lib):
    assert lib.dg_version() == 105
    for code, name in binding.STATUS_NAMES.items():
        assert lib.dg_status_string(code).decode().startswith(name)
    # the device-side group_offsets check has its own code, named in the header
    assert binding.STATUS_NAMES[7] == "DG_ERR_GROUP_OFFSETS"
    with open(os.path.join(ROOT, "include", "dg.h")) as f:
        assert "DG_ERR_GROUP_OFFSETS = 7" in f.read()


def test_host_validation_without_device(lib):
    null = ctypes.c_void_p(0)
    # shape errors and no-ops are decided before any CUDA call
    assert lib.dg_quantize_blockwise(null, 4, 17, null, null, null) == 2
    assert lib.dg_quantize_blockwise(null, -1, 16, null, null, null) == 2
    assert lib.dg_quantize_blockwise(null, 0, 16, null, null, null) == 0
    assert lib.dg_fp8_gemm_blockscaled(null, null, null, null, null, 8, 16, 100, null) == 2  # K % 16
    assert lib.dg_fp8_gemm_blockscaled(null, null, null, null, null, 8, 16, 112, null) == 1  # K tail ok
    assert lib.dg_fp8_grouped_gemm_contiguous(null, null, null, null, null, null, 128, 2, 128, 40, null) == 2
    assert lib.dg_fp8_gemm_blockscaled(null, null, null, null, null, 8, 24, 128, null) == 2  # N % 16
    assert lib.dg_fp8_gemm_blockscaled(null, null, null, null, null, 8, 16, 0, null) == 2    # K == 0
    assert lib.dg_fp8_gemm_blockscaled(null, null, null, null, null, 0, 16, 128, null) == 0  # M == 0
    assert lib.dg_fp8_gemm_blockscaled(null, null, null, null, null, 8, 16, 128, null) == 1  # null data
    assert lib.dg_fp8_gemm_blockscaled_select(null, null, null, null, null, 200, 16, 128, 2, null) == 2
    assert lib.dg_fp8_gemm_blockscaled_select(null, null, null, null, null, 20, 16, 128, 7, null) == 1
    assert lib.dg_fp8_grouped_gemm_contiguous(null, null, null, null, null, null, 100, 2, 128, 128, null) == 2
    assert lib.dg_fp8_grouped_gemm_contiguous(null, null, null, null, null, null, 128, 0, 128, 128, null) == 2
    assert lib.dg_fp8_grouped_gemm_contiguous(null, null, null, null, null, null, 128, 2, 64, 128, null) == 2
    assert lib.dg_fp8_grouped_gemm_contiguous(null, null, null, null, null, null, 0, 2, 128, 128, null) == 0
    assert lib.dg_fp8_grouped_gemm_contiguous(null, null, null, null, null, null, 128, 2, 128, 128, null) == 1
    # the BF16-activation GEMM: shapes first, then pointers
    assert lib.dg_fp8_gemm_blockscaled_bf16a(null, null, null, null, null, null, 8, 16, 100, null) == 2
    assert lib.dg_fp8_gemm_blockscaled_bf16a(null, null, null, null, null, null, 8, 24, 128, null) == 2
    assert lib.dg_fp8_gemm_blockscaled_bf16a(null, null, null, null, null, null, 0, 16, 128, null) == 0
    assert lib.dg_fp8_gemm_blockscaled_bf16a(null, null, null, null, null, null, 8, 16, 128, null) == 1
    # masked MoE: G in [1, 256], N % 128, K % 16, then pointers
    assert lib.dg_fp8_grouped_gemm_masked(null, null, null, null, null, null, 0, 128, 128, 128, null) == 2
    assert lib.dg_fp8_grouped_gemm_masked(null, null, null, null, null, null, 257, 128, 128, 128, null) == 2
    assert lib.dg_fp8_grouped_gemm_masked(null, null, null, null, null, null, 2, 128, 64, 128, null) == 2
    assert lib.dg_fp8_grouped_gemm_masked(null, null, null, null, null, null, 2, 128, 128, 40, null) == 2
    assert lib.dg_fp8_grouped_gemm_masked(null, null, null, null, null, null, 2, 0, 128, 128, null) == 0
    assert lib.dg_fp8_grouped_gemm_masked(null, null, null, null, null, null, 2, 128, 128, 128, null) == 1
    # masked-slab quantizer: G in [1, 1024], cols % 16, then pointers
    assert lib.dg_quantize_blockwise_masked(null, 0, 128, 16, null, null, null, null) == 2
    assert lib.dg_quantize_blockwise_masked(null, 1025, 128, 16, null, null, null, null) == 2
    assert lib.dg_quantize_blockwise_masked(null, 2, 128, 17, null, null, null, null) == 2
    assert lib.dg_quantize_blockwise_masked(null, 2, 0, 16, null, null, null, null) == 0
    assert lib.dg_quantize_blockwise_masked(null, 2, 128, 16, null, null, null, null) == 1
    # per-token scales
    assert lib.dg_quantize_1x128(null, 4, 17, null, null, null) == 2
    assert lib.dg_quantize_1x128(null, 0, 16, null, null, null) == 0
    assert lib.dg_fp8_gemm_1x128(null, null, null, null, null, 8, 16, 100, null) == 2
    assert lib.dg_fp8_gemm_1x128(null, null, null, null, null, 8, 16, 128, null) == 1
    assert lib.dg_fp8_gemm_1x128_select(null, null, null, null, null, 8, 16, 128, 2, null) == 1
    odd = ctypes.c_void_p(0x1001)
    assert lib.dg_fp8_gemm_blockscaled(odd, odd, odd, odd, odd, 8, 16, 128, null) == 3
    # misaligned pointers are refused before any CUDA call, on every entry point
    ok16 = ctypes.c_void_p(0x10000)
    assert lib.dg_quantize_blockwise(odd, 8, 16, ok16, ok16, null) == 3
    assert lib.dg_quantize_1x128(ok16, 8, 16, odd, ok16, null) == 3
    assert lib.dg_quantize_blockwise_masked(ok16, 2, 8, 16, odd, ok16, ok16, null) == 3
    assert lib.dg_quantize_blockwise_masked(odd, 2, 8, 16, ok16, ok16, ok16, null) == 3
    assert lib.dg_fp8_gemm_blockscaled_bf16a(odd, ok16, ok16, ok16, ok16, ok16, 8, 16, 128, null) == 3
    assert lib.dg_fp8_gemm_blockscaled_bf16a(ok16, ok16, ok16, ok16, odd, ok16, 8, 16, 128, null) == 3
    assert lib.dg_fp8_gemm_1x128(ok16, ok16, odd, ok16, ok16, 8, 16, 128, null) == 3
    assert lib.dg_fp8_grouped_gemm_contiguous(ok16, ok16, ok16, ok16, ok16, odd, 128, 2, 128, 128, null) == 3
    assert lib.dg_fp8_grouped_gemm_masked(ok16, ok16, ok16, ok16, ok16, odd, 2, 128, 128, 128, null) == 3
    assert lib.dg_fp8_grouped_gemm_masked(odd, ok16, ok16, ok16, ok16, ok16, 2, 128, 128, 128, null) == 3
    # an unknown kernel choice
    assert lib.dg_fp8_gemm_1x128_select(ok16, ok16, ok16, ok16, ok16, 8, 16, 128, 9, null) == 1
    # the fused one-launch form is a choice of the BF16-activation call only, up to M = 16
    fused = 4
    assert lib.dg_fp8_gemm_blockscaled_select(ok16, ok16, ok16, ok16, ok16, 8, 16, 128, fused, null) == 1
    assert lib.dg_fp8_gemm_1x128_select(ok16, ok16, ok16, ok16, ok16, 8, 16, 128, fused, null) == 1
    assert lib.dg_fp8_gemm_blockscaled_bf16a_select(ok16, ok16, ok16, ok16, ok16, ok16, 17, 16, 128, fused, null) == 2
    assert lib.dg_fp8_gemm_blockscaled_bf16a_select(ok16, ok16, ok16, ok16, ok16, ok16, 200, 16, 128, 2, null) == 2
    assert lib.dg_fp8_gemm_blockscaled_bf16a_select(ok16, ok16, ok16, ok16, ok16, ok16, 8, 16, 128, 9, null) == 1
    assert lib.dg_fp8_gemm_blockscaled_bf16a_select(odd, ok16, ok16, ok16, ok16, ok16, 8, 16, 128, fused, null) == 3
    assert lib.dg_fp8_gemm_blockscaled_bf16a_select(null, null, null, null, null, null, 0, 16, 128, fused, null) == 0


def declared_signatures():
    """{name: number of parameters} for every function include/dg.h declares."""
    text = open(os.path.join(ROOT, "include", "dg.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(dg_\w+)\s*\(([^()]*)\)\s*;", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else len(params.split(","))
    return out


def test_binding_argument_lists_match_the_header(lib):
    """A parameter added on one side only would shift every argument after it."""
    sigs = declared_signatures()
    assert set(sigs) == set(binding.EXPORTS)
    for name, n in sigs.items():
        argtypes = getattr(lib, name).argtypes
        if argtypes is not None:
            assert len(argtypes) == n, (name, len(argtypes), n)


def _ctype_of(param: str):
    p = param.strip()
    if "*" in p or p.startswith("cudaStream_t"):
        return ctypes.c_void_p
    base = p.rsplit(" ", 1)[0].replace("const ", "").strip()
    return {"int64_t": ctypes.c_int64, "uint64_t": ctypes.c_uint64, "int": ctypes.c_int,
            "dg_kernel_t": ctypes.c_int, "dg_status_t": ctypes.c_int}[base]


def test_binding_argument_types_match_the_header(lib):
    """Pointer, 32- and 64-bit integer parameters must be passed as such: an int64_t
    bound as c_int leaves the upper half of the register undefined."""
    text = open(os.path.join(ROOT, "include", "dg.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    for m in re.finditer(r"\b(dg_\w+)\s*\(([^()]*)\)\s*;", text):
        params = m.group(2).strip()
        if params in ("", "void"):
            continue
        want = [_ctype_of(x) for x in params.split(",")]
        got = list(getattr(lib, m.group(1)).argtypes)
        assert got == want, (m.group(1), got, want)
