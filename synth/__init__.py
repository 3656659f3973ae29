"""Seeded synthetic inputs for the SVDQuant W4A4 / AWQ W4A16 linear layers.

This package is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It holds no quantisation, packing or GEMM arithmetic: only
random draws (a counter-based splitmix64 generator with a Box-Muller normal
transform) and the layer-parameter recipe that stands in for a calibrated
checkpoint (smoothing vector and rank-r factors, see ``inputs``).
"""

from .inputs import (  # noqa: F401
    CONFIGS,
    config_layer,
    awq_inputs,
    qkv_epilogue_inputs,
    bf16_bits,
    bf16_bits_to_f32,
    normal,
    svdq_layer,
    uniform,
)
