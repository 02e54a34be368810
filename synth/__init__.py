"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This package holds input generation and workload tables only: no step of the
attention method (no partition, pooling, scoring, selection or attention
arithmetic) lives here.
"""
from .video_latents import (  # noqa: F401
    splitmix64_stream,
    uniform01,
    standard_normal,
    smooth_fields,
    make_qkv,
    make_dout,
    seed_for,
)
from .workloads import BOXES_8_48_72, PAPER_10_48_60, WORKLOADS, Workload  # noqa: F401
