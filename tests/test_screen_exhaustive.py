"""The CUDA quantizer's E4M3 conversion screen, restated in C and checked over every
FP32 value it can meet (tests/native/screen_exhaustive.c; about 2.3e9 values,
multithreaded): when the screen lets y = x * RN(1/s) through, y and RN(x / s) give
the same E4M3 code.  With the GPU parity tests of the quantizer (bit-identical to
the oracle's division on every input tried) this is the argument that the fast path
is exact."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_screen_is_sound_on_all_fp32_values(tmp_path):
    exe = tmp_path / "screen_exhaustive"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-o", str(exe),
                    os.path.join(HERE, "native", "screen_exhaustive.c"), "-lm"], check=True)
    p = subprocess.run([str(exe)], capture_output=True, text=True, timeout=1200)
    assert p.returncode == 0 and p.stdout.strip().endswith("counterexamples 0"), p.stdout[-2000:]
