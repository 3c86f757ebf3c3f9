"""CPU oracle of the CommunityKV decode step (float64, numpy).

Test infrastructure only: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg, never by the library or its binding.
"""
from .ckv_oracle import *  # noqa: F401,F403
