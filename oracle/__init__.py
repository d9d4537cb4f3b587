"""CPU oracle for the ETA decode step (test infrastructure only).

Only the test suite, the package's smoke check and the benchmark's CPU-baseline
leg may import this package.  It does not import the CUDA library.
"""
from .eta_oracle import *  # noqa: F401,F403
