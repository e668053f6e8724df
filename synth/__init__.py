"""Seeded synthetic inputs for compressed-KV decode attention.

This package only draws random numbers and casts them to the storage dtype.
It holds none of the compression or attention arithmetic, so both the CPU
oracle and the CUDA path can take their inputs from it.
"""
from .workloads import (  # noqa: F401
    WORKLOADS,
    Workload,
    bf16_bits_to_f64,
    block_taus,
    f64_to_bf16_bits,
    gen_block_f64,
    gen_layer,
    gen_pool_f64,
    gen_queries,
    gen_suffix,
    outlier_scales,
    to_storage,
    from_storage,
)
