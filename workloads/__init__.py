"""Seeded synthetic workloads (shapes, distributions, planted keys) shared by the
oracle side and the CUDA side of the tests and the benchmark."""
from . import configs, make, rng  # noqa: F401
