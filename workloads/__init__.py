"""Seeded synthetic inputs for the SparseGPT layer solver.

This package only draws numbers: weights W, calibration activations X and the
per-channel scales that shape X. It holds none of the pruning method's
arithmetic, so both the double-precision oracle (through the tests) and the
CUDA path (through the tests, the bench and the smoke check) can consume the
same bytes without sharing any solver code.
"""

from .gen import (  # noqa: F401
    CONFIGS,
    LayerSpec,
    bf16_bits_to_f64,
    channel_scales,
    gen_weights,
    gen_activations,
    normals,
)
