"""CPU oracle for the FP8 (E4M3) 128x128 block-scaled GEMM and its block quantizer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import, call, link or run anything in this
package.  It shares no code with the CUDA library and never imports it.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import BLK, RTOL, ATOL_RMS, num_threads  # noqa: F401
