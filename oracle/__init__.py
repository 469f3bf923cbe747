"""Float64 CPU oracle for BCJR-QAT (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  It shares no code with the CUDA library.

  bcjr_oracle.c  -- the unfactored float64 forward-backward, its adjoint, the
                    max-sum hard decode and the dense transfer-matrix variant
  brute.py       -- enumeration of every trellis path on tiny problems
"""
from .clib import (  # noqa: F401
    build,
    forward,
    backward,
    viterbi,
    alpha_beta,
    dense_forward,
    dense_backward,
    max_threads,
)
