"""Seeded synthetic workloads: generators, shapes and inputs (no arithmetic of the method)."""
from . import configs, gen, inputs  # noqa: F401
