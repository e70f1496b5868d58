"""fp64 CPU oracle of the hybrid-head layer — test infrastructure only.

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package; the CUDA library neither calls nor links it.
"""
from . import hymba_oracle  # noqa: F401
from .hymba_oracle import Spec  # noqa: F401
