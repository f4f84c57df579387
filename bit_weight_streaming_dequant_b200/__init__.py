"""libq4dec: Q4_0 decode hot path (dequant-fused GEMV and Q4-KV decode
attention) for NVIDIA B200, exported through a C ABI (include/q4dec.h).

``bit_weight_streaming_dequant_b200.q4dec`` is the Python binding;
``bit_weight_streaming_dequant_b200.build`` compiles the library in-tree.
"""
from .q4dec import (  # noqa: F401
    Q4DecError,
    q4_gemv,
    q4kv_attn_decode,
    plan_gemv,
    plan_attn,
    device_error,
    lib,
)
