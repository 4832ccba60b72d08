"""Float64 CPU oracle of the POET-X layer.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the package smoke
check and the benchmark's CPU-baseline / reference legs, never by the
library.  It shares no code with the CUDA path.
"""
from .poetx_oracle import *  # noqa: F401,F403
from .splitmix import (mix64, splitmix_output, splitmix_stream,  # noqa: F401
                       permutation_keys, resample_permutation)
