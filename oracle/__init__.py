"""CPU oracle for the weight-only-quantized linear layer (test infrastructure).

Plain, slow, fp64 NumPy code that states what the layer computes, written from
the pages' definitions.  It reads the canonical layouts produced by
``synth`` and shares nothing with the CUDA library: no kernels, headers,
packers, tables or helpers.  Only the tests, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it; the library itself never
does, and nothing in the product path falls back to it.
"""
from .qlinear_oracle import *  # noqa: F401,F403
