"""Shared test helpers: cached seeded layers and the parity check."""
import functools

import numpy as np

import oracle
from synth import gen

# relative L2 error and max-abs error (relative to max |y_ref|) allowed for fp16 outputs
# computed with fp32 accumulation (fp16 rounding of y alone contributes <= 2^-11 relative)
REL_L2_TOL = 2e-3
MAX_ABS_TOL = 1e-2


def assert_parity(y_gpu, y_ref, per_row=True, what=""):
    y = np.asarray(y_gpu, dtype=np.float64)
    r = np.asarray(y_ref, dtype=np.float64)
    rel, mabs = oracle.parity_errors(y, r)
    assert rel <= REL_L2_TOL and mabs <= MAX_ABS_TOL, f"{what}: relL2={rel:.3e} maxabs={mabs:.3e}"
    if per_row and y.ndim == 2 and y.shape[0] > 1:
        for m in range(y.shape[0]):
            rel, mabs = oracle.parity_errors(y[m], r[m])
            assert rel <= REL_L2_TOL and mabs <= MAX_ABS_TOL, \
                f"{what} row {m}: relL2={rel:.3e} maxabs={mabs:.3e}"


@functools.lru_cache(maxsize=8)
def uniform_layer(seed, K, N, bits):
    return gen.uniform_layer(seed, K, N, bits)


@functools.lru_cache(maxsize=4)
def lut4_layer(seed, K, N):
    return gen.lut4_layer(seed, K, N)


@functools.lru_cache(maxsize=4)
def outlier_layer(seed, K, N):
    return gen.outlier_layer(seed, K, N)
