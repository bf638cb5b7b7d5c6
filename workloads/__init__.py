"""Seeded synthetic workloads (geometry, seeds, input generators).

Shared by the oracle tests and the CUDA path; holds none of the method's
arithmetic.
"""
from .configs import Workload, ALL, BY_NAME, TINY, FRAME_TILE, DITANGO_REUSE, LONG_VIDEO, DENSE, scaled  # noqa: F401
