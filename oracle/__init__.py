"""CPU oracle for the ReSpinQuant boundary path (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline / reference
leg may import this package. The CUDA library never does, and this package
never imports the library.
"""
from .respin_oracle import *  # noqa: F401,F403
