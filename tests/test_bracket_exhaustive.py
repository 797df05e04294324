"""The CUDA quantizer's E4M3 conversion, restated in C and checked for every pair it
can meet (tests/native/bracket_exhaustive.c): every positive finite BF16 block amax
(so every possible scale s = fl32(amax / 448)) against every BF16 x with
|x| <= amax, about 1.07e9 pairs.  The code decided from the two bracketing products
(or the division they fall back to) must equal E4M3(fl32(x / s)) in every case."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_conversion_is_exact_for_every_bf16_value_and_block_scale(tmp_path):
    exe = tmp_path / "bracket_exhaustive"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-o", str(exe),
                    os.path.join(HERE, "native", "bracket_exhaustive.c"), "-lm"], check=True)
    p = subprocess.run([str(exe)], capture_output=True, text=True, timeout=1200)
    assert p.returncode == 0 and p.stdout.strip().endswith("mismatches 0"), p.stdout[-2000:]
