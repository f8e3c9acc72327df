"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This package holds workload shapes, method settings and the video-grid input
generator.  It contains none of the attention method's arithmetic, so both the
oracle and the CUDA path may import it without sharing method code.
"""

from .workloads import WORKLOADS, Workload, get_workload  # noqa: F401
from .video_grid import generate_head, generate_inputs, bf16_round, drift_inputs  # noqa: F401
