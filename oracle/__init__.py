"""fp64 CPU oracle for the Kimi Delta Attention recurrence.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA library.
"""
from .kda_oracle import (OracleLib, backward, build, decode_step, default, forward,
                         num_threads)

__all__ = ["OracleLib", "backward", "build", "decode_step", "default", "forward",
           "num_threads"]
