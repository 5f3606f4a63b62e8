"""Oracle: a plain, slow FP64 CPU statement of the NVFP4 weight-only routed-expert MoE layer.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this package.  It shares no code with the CUDA library (no
kernels, headers, tables, constants or pre/post-processing); both sides meet only in the
seeded input generators of ``moe_inputs``, which hold none of the layer's arithmetic.

Sources (pages on Reflection's Beam-1.0-501B-A23B; cited by page title and section):
  * "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents",
    section "What this pack holds": one record per (layer, expert) holds gate, up and down,
    each as E2M1 codes in U32 words, one E4M3 block scale per 16 inputs and one F32 global
    scale; MLX forms a block's scale as e4m3(block scale) x (g / 2688) in f32; the 256
    routed experts with 8 active per token; activations stay BF16.
  * "Beam-1.0-501B-A23B VQ GGUF", section "What stays native": router logits and SwiGLU
    are FP32 numerics in the source model (the oracle computes both in FP64).
  * The method statement this library implements: top-k over the router logits with ties
    to the lower expert index, softmax over the k selected logits, SwiGLU experts
    (gate/up/down), a weighted combine, and, for stacked layers, a residual add.

Parity pins: every function here is checked in tests/test_oracle_*.py against library
routines (ml_dtypes, torch), closed forms, brute force and the record geometry that the
streaming-pack page prints.  Absolute layer outputs have no worked example on the pages;
they rest on those pins (see the module docstrings).
"""
from .nvfp4 import (  # noqa: F401
    e2m1_value,
    e4m3_value,
    E2M1_VALUES,
    E4M3_VALUES,
    projection_bytes,
    decode_codes,
    global_multiplier,
    dequant,
    read_record,
)
from .moe import (  # noqa: F401
    route,
    permute,
    silu,
    expert_forward,
    expert_forward_w4a4,
    layer_forward,
    bf16_bits_to_f64,
    round_to_bf16_bits,
    residual_add,
)
from .sources import GeneratedRecords  # noqa: F401
from .encode import (  # noqa: F401
    e2m1_round,
    e4m3_round,
    tensor_global,
    encode_projection,
    encode_f32,
    quantize_rows,
    quantize_static,
    decode_blocks,
    pack_codes,
)
