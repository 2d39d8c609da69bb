"""Pins of the oracle's codebook GEMV (CodeGEMM m1v4g128) against facts that do not
come from the oracle.

* a hand-derived closed form (all-ones x, one code everywhere);
* exact rational brute force on a tiny layer, codes read straight from the arrays;
* a codebook whose centroids are the 2-bit digits of their index reduces the
  format to W2 uniform quantization with zero point 0 (a separately pinned function);
* one-hot activations reproduce one dequantized weight row;
* the Psumbook evaluation agrees with the eager dequantize-then-dot form within fp64
  rounding (two different orders of the same sum);
* the nearest-centroid generator really picks the nearest centroid;
* planted mistakes (vector/element index swapped, wrong scale group, transposed codes)
  fail these pins.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from synth import gen

V, G128 = 4, 128


def test_closed_form_all_ones():
    """x = 1, every code 5, C[5] = (0.5, -0.25, 1, 0), s = 2: each 4-vector contributes
    2 * 1.25 = 2.5, and K = 256 has 64 vectors: y = 160 in every column."""
    K, N = 256, 3
    C = np.zeros((256, 4), dtype=np.float16)
    C[5] = [0.5, -0.25, 1.0, 0.0]
    codes = np.full((K // V, N), 5, dtype=np.uint8)
    s = np.full((K // G128, N), 2.0, dtype=np.float16)
    x = np.ones((1, K), dtype=np.float16)
    assert np.all(oracle.gemv_codebook(x, codes, C, s, V, G128) == 160.0)
    assert np.all(oracle.gemv_codebook_psumbook(x, codes, C, s, V, G128) == 160.0)


def test_bruteforce_rationals():
    K, N, M = 256, 5, 2
    L = gen.codebook_layer(41, K, N)
    x = gen.activations(41, M, K)
    y = oracle.gemv_codebook(x, L.codes, L.codebook, L.scales, V, G128)
    yp = oracle.gemv_codebook_psumbook(x, L.codes, L.codebook, L.scales, V, G128)
    for m in range(M):
        for n in range(N):
            exact = Fraction(0)
            for k in range(K):
                code = int(L.codes[k // 4, n])
                w = Fraction(float(L.scales[k // 128, n])) * Fraction(float(L.codebook[code, k % 4]))
                exact += Fraction(float(x[m, k])) * w
            tol = Fraction(1, 2 ** 40) * (1 + abs(exact))
            assert abs(Fraction(float(y[m, n])) - exact) <= tol
            assert abs(Fraction(float(yp[m, n])) - exact) <= tol


def test_digit_codebook_reduces_to_w2_uniform():
    K, N, M = 384, 24, 3
    C = np.array([[(i >> (2 * t)) & 3 for t in range(4)] for i in range(256)], dtype=np.float16)
    rs = np.random.default_rng(9)
    codes = rs.integers(0, 256, size=(K // V, N), dtype=np.uint8)
    digits = np.empty((K, N), dtype=np.uint8)
    for t in range(4):
        digits[t::4] = (codes >> (2 * t)) & 3
    s = (0.01 + 0.05 * rs.random((K // G128, N))).astype(np.float16)
    z = np.zeros_like(s)
    x = gen.activations(9, M, K)
    y = oracle.gemv_codebook(x, codes, C, s, V, G128)
    yu = oracle.gemv_uniform(x, gen.pack_codes(digits, 2), s, z, 2, G128)
    assert np.allclose(y, yu, rtol=1e-12, atol=1e-12)


def test_one_hot_and_psumbook_agreement():
    K, N = 512, 40
    L = gen.codebook_layer(43, K, N)
    x = np.zeros((1, K), dtype=np.float16)
    k0 = 301
    x[0, k0] = 1
    y = oracle.gemv_codebook(x, L.codes, L.codebook, L.scales, V, G128)[0]
    want = L.scales[k0 // 128].astype(np.float64) * \
        L.codebook[L.codes[k0 // 4], k0 % 4].astype(np.float64)
    assert np.array_equal(y, want)
    xr = gen.activations(43, 4, K)
    a = oracle.gemv_codebook(xr, L.codes, L.codebook, L.scales, V, G128)
    b = oracle.gemv_codebook_psumbook(xr, L.codes, L.codebook, L.scales, V, G128)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)
    cols = [3, 39, 0]
    assert np.array_equal(oracle.gemv_codebook(xr, L.codes, L.codebook, L.scales, V, G128, cols),
                          a[:, cols])


def test_nearest_centroid_generator():
    K, N = 256, 8
    w = gen.weights(44, K, N)
    L = gen.codebook_layer(44, K, N, w=w)
    s = L.scales.astype(np.float64)
    C = L.codebook.astype(np.float64)
    for n in range(N):
        for j in range(0, K // 4, 7):
            u = w[4 * j:4 * j + 4, n].astype(np.float64) / s[(4 * j) // 128, n]
            d = ((C - u[None, :]) ** 2).sum(axis=1)
            assert d[L.codes[j, n]] == d.min()
    # the format represents the weights within the nearest-centroid distance times s
    deq = oracle.dequant_codebook(L.codes, L.codebook, L.scales, V, G128)
    assert np.all(np.abs(deq - w) <= np.repeat(s, 128, axis=0) * 2 + 1e-12)


# ---------------------------------------------------------------------------
# planted mistakes


def _mut_index_swap(codes, codebook, scales, v, group, cols=None):
    c = codes if cols is None else codes[:, cols]
    s = (scales if cols is None else scales[:, cols]).astype(np.float64)
    Cb = codebook.astype(np.float64)
    k = np.arange(c.shape[0] * v)
    return s[k // group, :] * Cb[c[k % c.shape[0], :], (k // c.shape[0] % v)[:, None]]


def _mut_scale_group(codes, codebook, scales, v, group, cols=None):
    c = codes if cols is None else codes[:, cols]
    s = (scales if cols is None else scales[:, cols]).astype(np.float64)
    Cb = codebook.astype(np.float64)
    k = np.arange(c.shape[0] * v)
    return s[(k // group + 1) % s.shape[0], :] * Cb[c[k // v, :], (k % v)[:, None]]


def _mut_element_order(codes, codebook, scales, v, group, cols=None):
    c = codes if cols is None else codes[:, cols]
    s = (scales if cols is None else scales[:, cols]).astype(np.float64)
    Cb = codebook.astype(np.float64)
    k = np.arange(c.shape[0] * v)
    return s[k // group, :] * Cb[c[k // v, :], (v - 1 - k % v)[:, None]]


@pytest.mark.parametrize("mutant", [_mut_index_swap, _mut_scale_group, _mut_element_order])
def test_mutants_fail(monkeypatch, mutant):
    from oracle import qlinear_oracle as qo
    monkeypatch.setattr(qo, "dequant_codebook", mutant)
    failed = 0
    for pin in (test_closed_form_all_ones, test_bruteforce_rationals,
                test_digit_codebook_reduces_to_w2_uniform, test_one_hot_and_psumbook_agreement):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1
