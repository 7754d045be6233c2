"""CPU fp64 oracle for DSA decode.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package.  The CUDA library never calls it and
shares no code with it.
"""
from .dsa_oracle import *  # noqa: F401,F403
from .hisparse import PAGE_TOKENS as TIER_PAGE_TOKENS, TierOracle, TierOverflow  # noqa: F401
