"""Seeded synthetic inputs for the LISA attention layer.

This package holds the workload shapes and the deterministic input generators
that both the fp64 oracle (``oracle/``) and the CUDA path consume.  It contains
none of the method's arithmetic: only random draws, the rounding of those draws
to the storage dtype, and array layout.
"""

from .configs import CONFIGS, LisaConfig, get_config
from .gen import (
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    round_to_dtype,
    make_rng,
    gen_layer,
    gen_step,
    gen_lengths,
    LayerData,
    StepData,
)

__all__ = [
    "CONFIGS",
    "LisaConfig",
    "get_config",
    "bf16_bits_to_f32",
    "f32_to_bf16_bits",
    "round_to_dtype",
    "make_rng",
    "gen_layer",
    "gen_step",
    "gen_lengths",
    "LayerData",
    "StepData",
]
