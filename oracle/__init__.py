"""CPU oracle for the Q4_0 decode path (and the Q8_0 K/V cache variant) (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
and reference legs) may import this package.  The library's product path never
calls it, and it shares no code with the CUDA path.
"""
from .q4_oracle import (  # noqa: F401
    bf16_bits_to_f64,
    f16_bits_to_f64,
    unpack_superblocks,
    dequant,
    unpack_q8_superblocks,
    dequant_q8,
    dequant_weights,
    weight_rows,
    gemv,
    gemv_tolerance,
    attn_probs,
    attn_decode,
    quantize_q4_0_rows,
    silu,
    silu_prime,
    SILU_PRIME_CRIT,
    silu_prime_max,
    SWIGLU_EPILOGUE_REL,
    swiglu_tolerance,
    gemv_swiglu,
    kv_append,
)
