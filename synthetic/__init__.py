"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This package holds only input generation (smooth random Fourier fields plus
noise, a per-token difficulty score) and the workload table.  It contains none
of the attention or selector arithmetic: both the CUDA library and the fp64
oracle receive what it produces as plain inputs.
"""
from .fields import make_qkv, make_difficulty
from .workloads import WORKLOADS, workload

__all__ = ["make_qkv", "make_difficulty", "WORKLOADS", "workload"]
