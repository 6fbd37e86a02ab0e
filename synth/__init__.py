"""Seeded synthetic inputs shared by the CPU oracle, the tests and the benchmark.

This package only draws random numbers and lays out frames in time order. It holds none
of the method's arithmetic (no attention, no statistics, no solve), so that the oracle and
the CUDA path can both read the same bytes without sharing any computation.
"""
from .workload import (  # noqa: F401
    IspaConfig,
    CONFIGS,
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    frame_kv,
    chunk_q,
    w_out,
    chunk_layout,
    cache_frames,
    make_rng,
    kv_tensor,
    normal_tensor,
)
