"""Seeded synthetic workloads and inputs (no part of the MoE layer's arithmetic)."""
from . import gen, workloads  # noqa: F401
