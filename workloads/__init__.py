"""Synthetic DSA workloads: the five configurations and their seeded input generators.

This package holds shapes and random numbers only -- none of the method's arithmetic --
so both the CUDA library's tests/benchmark and the CPU oracle's checks can share it.
"""
from .configs import CONFIGS, DSAConfig, get_config  # noqa: F401
from .gen import dsa_inputs, swa_inputs  # noqa: F401
