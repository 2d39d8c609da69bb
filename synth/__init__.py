"""Seeded synthetic inputs for the weight-only-quantized GEMV workloads.

This package produces the *inputs* of the quantized linear layer: random
weights, their low-bit codes in the canonical layouts, quantization parameters,
Tile-COO outlier arrays and fp16 activations. It is shared by the tests, the
benchmark and the oracle's checks, and it contains none of the layer's own
arithmetic (no unpacking, dequantization or dot products).
"""
from .gen import *  # noqa: F401,F403
