"""Seeded synthetic MSA workloads (inputs only; no part of the method)."""
from . import gen, configs  # noqa: F401
