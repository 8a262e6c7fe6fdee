"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This package draws random numbers and lays them out as tensors of the
workload shapes; it holds none of the method's arithmetic (no pruning, no
selection, no GEMM).  See ``workload.gen`` for the generator definition.
"""
from .gen import (  # noqa: F401
    CONFIGS,
    Config,
    fnv1a64,
    splitmix64_stream,
    uniform01,
    normal,
    f32_to_f16,
    f32_to_bf16_bits,
    bf16_bits_to_f32,
    make_inputs,
    tw_tile_counts,
)
