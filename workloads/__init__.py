"""Seeded synthetic workloads for the MiniMax-H3 block forward.

This package only draws random numbers and builds packed layouts (row tags,
(t, h, w) positions, timestep indices, index tensors). It holds none of the
block's arithmetic, so both the CPU oracle and the CUDA path can take their
inputs from it without sharing any part of the computation.
"""

from .h3_workloads import (  # noqa: F401
    Dims,
    TINY_DIMS,
    FULL_DIMS,
    Layout,
    BlockWeights,
    PrologueWeights,
    TAG_VIDEO,
    TAG_TEXT,
    TAG_AUDIO,
    TAG_PAD,
    f32_to_bf16_bits,
    bf16_bits_to_f32,
    normal_bf16,
    make_layout,
    config_layout,
    config_dims,
    random_layout,
    block_weights,
    prologue_weights,
    activations,
    CONFIG_NAMES,
    DenoiserWeights,
    denoiser_weights,
    denoiser_inputs,
    random_code_bytes,
    random_scales,
)
