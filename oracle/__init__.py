"""fp64 CPU oracle for the HSTU layer (test infrastructure only).

Only tests, the smoke check and the benchmark's CPU-baseline leg import this
package.  It shares no code with the CUDA library or its binding.
"""
from .hstu_oracle import *  # noqa: F401,F403
