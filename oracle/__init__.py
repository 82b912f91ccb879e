"""CPU oracle for head-wise hybrid attention (test infrastructure only).

This package is the slow, plain reference that the CUDA library is checked
against. Only the tests, the smoke check and the benchmark's CPU-baseline leg
may import it; the library itself never does. It shares no code with the
CUDA sources.
"""
from .rtp_oracle import *  # noqa: F401,F403
