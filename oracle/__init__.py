"""The fp64 CPU oracle of the LSH attention forward pass.

Test infrastructure: imported only by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA library or its binding.
"""
from .lsh_oracle import *  # noqa: F401,F403
from .lsh_oracle import SELF_SCORE  # noqa: F401
