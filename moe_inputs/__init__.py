"""Seeded synthetic inputs for the NVFP4 weight-only routed-expert MoE layer.

This package is shared by the CPU oracle's tests, the GPU parity tests and the benchmark.
It only draws random bytes, normal deviates and router logits and writes them in the
expert-record layout; it performs none of the layer's arithmetic (no decoding of codes or
scales, no routing, no products, no rounding of results).
"""
from .gen import (  # noqa: F401
    CONFIGS,
    LayerConfig,
    RecordLayout,
    record_layout,
    record_bytes,
    bank_host,
    make_x,
    make_x_wide,
    make_logits,
    make_act_scales,
    sample_tokens,
    disjoint_routing_logits,
    global_value,
)
