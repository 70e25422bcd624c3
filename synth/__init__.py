"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This package holds random-number draws and data-representation helpers only
(bf16 rounding of generated values); none of the quantisation, smoothing,
low-rank or GEMM arithmetic lives here.
"""
from .inputs import *  # noqa: F401,F403
