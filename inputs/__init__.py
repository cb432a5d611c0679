"""Seeded synthetic inputs shared by the oracle-side tests and the CUDA-side tests/bench.

This package holds no arithmetic of the quantization method: it only draws fp16
weight and activation tensors with the shapes and value distributions of the
GLM-130B projection layers. See :mod:`inputs.synthetic`.
"""
from .synthetic import (  # noqa: F401
    GLM_PROJECTIONS,
    PROJECTION_ORDER,
    TINY_N,
    TINY_K,
    TINY_M,
    gaussian_fp16,
    tiny_weight,
    tiny_activations,
    projection_weight,
    decode_activations,
    prefill_activations,
    outlier_positions,
    outlier_activations,
)
