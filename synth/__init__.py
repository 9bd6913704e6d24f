"""Seeded synthetic inputs for the quantized expert FFN layer.

This package is the only code that both the CPU oracle (``oracle/``) and the
CUDA library path consume.  It draws random bytes and random numbers and holds
none of the layer's arithmetic: no dequantisation, routing, SwiGLU or combine.
"""
from .generate import (  # noqa: F401
    CONFIGS,
    LayerConfig,
    block_bytes,
    expert_codes,
    expert_scales,
    layer_weights,
    mix32,
    router_bias,
    router_weights,
    tokens_bf16,
)
