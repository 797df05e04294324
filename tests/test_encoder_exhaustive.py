"""The oracle's E4M3 encoder against an independently written one, over every finite
FP32 bit pattern (tests/native/encoder_exhaustive.c; ~4.3e9 values, multithreaded C)."""
import os
import shutil
import subprocess

import pytest

from oracle import build as obuild

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_encoder_agrees_on_all_finite_fp32_patterns(tmp_path):
    lib = obuild.build()  # oracle/libdg_oracle.so
    exe = tmp_path / "encoder_exhaustive"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-o", str(exe),
                    os.path.join(HERE, "native", "encoder_exhaustive.c"), lib, "-lm",
                    f"-Wl,-rpath,{os.path.dirname(lib)}"], check=True)
    p = subprocess.run([str(exe)], capture_output=True, text=True, timeout=1200)
    assert p.returncode == 0 and p.stdout.strip().endswith("mismatches 0"), p.stdout[-2000:]
