"""Seeded synthetic inputs for the LiftQuant lift-then-project layer.

This package draws random tensors only. It holds none of the method's
arithmetic (no packing, whitening, lifting or contraction), so that both
the float64 oracle and the CUDA path can consume the same buffers without
sharing any computation.
"""

from .inputs import (  # noqa: F401
    CONFIGS,
    KronFactors,
    LayerConfig,
    LayerInputs,
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    make_kron_factors,
    make_layer,
    make_signs_pm1,
    make_packed_random,
    make_u_bf16,
    make_u_f32,
    rng_for,
)
