"""Seeded synthetic inputs for the sparse MLA prefill attend block.

This package only draws random numbers and lays them out; it holds none of
the attention arithmetic. Both the CPU oracle (through the tests) and the
CUDA library consume exactly the bytes it produces.
"""
from .inputs import (  # noqa: F401
    CONFIGS,
    D_LATENT,
    D_MODEL,
    D_NOPE,
    D_ROPE,
    D_V,
    SOFTMAX_SCALE,
    DecodeInputs,
    MlaInputs,
    decode_topk,
    make_decode_inputs,
    make_inputs,
    make_topk,
    quantize_e4m3_block128,
    sample_rows,
)
