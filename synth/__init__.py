"""Seeded synthetic workloads shared by the oracle-side tests and the GPU side."""

from . import configs, generate  # noqa: F401
