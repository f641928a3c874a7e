"""fp64 CPU oracle for the mask-free spatially adaptive DiT attention path.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg.  The product package never imports it.
"""
from .oracle import *  # noqa: F401,F403
