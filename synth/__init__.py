"""Seeded synthetic inputs shared by the oracle-side tests and the GPU path."""
from . import gen, configs  # noqa: F401
