"""Seeded synthetic inputs shared by the CPU oracle and the CUDA library's tests.

Holds only random-number generation and workload shapes: no quantisation,
routing or matrix arithmetic of the method.
"""
from .philox import philox4x32_10  # noqa: F401
from . import configs, draws  # noqa: F401
