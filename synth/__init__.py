"""Seeded synthetic inputs for the DELTA decode stack (shared by the oracle side and the GPU side).

Holds no attention arithmetic: only counter-based random numbers, the workload
definitions and the host-side construction of page tables, queries and planted
salient keys.
"""
from . import rng, configs  # noqa: F401
