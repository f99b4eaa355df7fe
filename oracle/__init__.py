"""CPU oracle for the single-stream DiT hot path (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg may
import this package.  The CUDA library never depends on it.
"""
from .zdit_oracle import *  # noqa: F401,F403
