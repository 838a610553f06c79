"""Seeded synthetic input generators shared by the oracle side and the GPU side.

This package holds random-number generation and the input recipes only; it has
no part of the HiLS computation.
"""
from .philox import philox4x32_10, gaussian_at, gaussian_range, uniform_at  # noqa: F401
from .workloads import WORKLOADS, Workload  # noqa: F401
