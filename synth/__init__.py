"""Seeded synthetic inputs shaped like the JetBlock workloads.

This package is shared by the float64 oracle side and the CUDA side: it draws
random numbers, applies the input distributions (sigmoid / softplus of normal
draws, unit-norm q and k, 1/fan_in weight scale) and rounds to the storage
dtype. It holds none of the mixer's arithmetic.
"""
from .jetblock import (  # noqa: F401
    JetShape,
    CONFIGS,
    bf16_bits_from_f64,
    bf16_bits_to_f64,
    prefill_inputs,
    prefill_inputs_blocked,
    decode_inputs,
    decode_inputs_blocked,
    spread_qk_norms,
    to_f64,
)
