"""Pins of the oracle's stand-alone dequantization (fp16 weights, ``[N, K]``) and of
its prefill matmul, against facts that do not come from the oracle.

* an exact-rational round-to-nearest-even into a binary format, written here from
  the IEEE 754 definition (significand width, exponent range, ties to even), so
  the pins do not re-call the NumPy casts the oracle uses;
* hand-derived fp16 bit patterns: a tie that rounds to even, overflow to
  infinity, subnormal scales, a zero difference;
* the LUT4 reading (the fp32 product stored as fp16): a hand-built case whose
  exact product rounds differently when rounded once to fp16;
* brute force with exact rationals on tiny non-square layers (a transposed or
  misindexed output fails);
* the prefill matmul: one-hot activations reproduce one weight column, brute
  force on a tiny case, and closeness to the exact-weight GEMV within the fp16
  rounding of the weights.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from synth import gen


def _rne(fr: Fraction, p: int, emin: int, emax: int) -> Fraction:
    """Round an exact rational to the binary format with p-bit significands and
    normal exponents emin..emax (subnormals below 2^emin), ties to even; values at
    or beyond max + half an ulp become +-inf (returned as None)."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, emin)                       # subnormals share the emin spacing
    ulp = Fraction(2) ** (e - (p - 1))
    q, r = divmod(a, ulp)
    q = int(q)
    if r * 2 > ulp or (r * 2 == ulp and q % 2 == 1):
        q += 1
    v = q * ulp
    max_finite = (2 - Fraction(2) ** (1 - p)) * Fraction(2) ** emax
    if v > max_finite:
        return None
    return sign * v


def _fp16(fr):
    return _rne(fr, 11, -14, 15)


def _fp32(fr):
    return _rne(fr, 24, -126, 127)


def _bits16(v) -> int:
    return int(np.array(v, dtype=np.float16).view(np.uint16))


def _expected_bits16(fr) -> int:
    r = _fp16(fr)
    if r is None:
        return 0x7C00 if fr > 0 else 0xFC00
    return _bits16(float(r))


# ---------------------------------------------------------------------------
# the rounding routine itself, on values whose fp16 encodings are known by hand


def test_rne_routine_hand_values():
    assert _fp16(Fraction(1)) == 1
    assert _fp16(Fraction(1) + Fraction(1, 2048)) == 1                     # tie -> even
    assert _fp16(Fraction(1) + Fraction(3, 2048)) == 1 + Fraction(2, 1024)  # tie -> even
    assert _fp16(Fraction(65504)) == 65504
    assert _fp16(Fraction(65519)) == 65504
    assert _fp16(Fraction(65520)) is None                                  # overflow
    assert _fp16(Fraction(1, 2 ** 25)) == 0                                # tie to even 0
    assert _fp16(Fraction(3, 2 ** 25)) == Fraction(2, 2 ** 24)
    assert _fp32(Fraction(1) + Fraction(1, 2 ** 24)) == 1


# ---------------------------------------------------------------------------
# uniform formats


def _uniform_from(codes, scales, zeros, bits):
    return gen.pack_codes(codes.astype(np.uint8), bits), scales, zeros


def test_uniform_fp16_hand_worked_bits():
    K, N = 128, 6
    bits = 4
    codes = np.zeros((K, N), dtype=np.uint8)
    scales = np.ones((1, N), dtype=np.float16)
    zeros = np.zeros((1, N), dtype=np.float16)
    # column 0: s = fp16(0.1) = 0x2E66, q - z = 3 -> exact 0.2999267578125 is the midpoint
    # of 0x34CC and 0x34CD; ties to even give 0x34CC
    scales[0, 0] = np.array(0x2E66, dtype=np.uint16).view(np.float16)
    codes[:, 0] = 3
    # column 1: s = 65504 (max fp16), q - z = 2 -> 131008 overflows to +inf (0x7C00)
    scales[0, 1] = np.float16(65504)
    codes[:, 1] = 2
    # column 2: same scale, q - z = -2 -> -inf (0xFC00)
    scales[0, 2] = np.float16(65504)
    codes[:, 2] = 1
    zeros[0, 2] = 3
    # column 3: smallest subnormal scale 2^-24 (0x0001), q - z = -3 -> 0x8003
    scales[0, 3] = np.array(1, dtype=np.uint16).view(np.float16)
    codes[:, 3] = 5
    zeros[0, 3] = 8
    # column 4: q = z -> +0
    scales[0, 4] = np.float16(0.75)
    codes[:, 4] = 9
    zeros[0, 4] = 9
    # column 5: s = 0.75, q - z = 15 - 0 -> 11.25 exactly (0x49A0)
    scales[0, 5] = np.float16(0.75)
    codes[:, 5] = 15
    qw, s, z = _uniform_from(codes, scales, zeros, bits)
    with np.errstate(over="ignore"):
        w = oracle.dequant_uniform_fp16_nk(qw, s, z, bits, 128)
    assert w.shape == (N, K) and w.dtype == np.float16
    got = w.view(np.uint16)[:, 0]
    assert list(got) == [0x34CC, 0x7C00, 0xFC00, 0x8003, 0x0000, 0x49A0]
    assert np.all(w.view(np.uint16) == got[:, None])  # every k of a column alike


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_uniform_fp16_bruteforce(bits):
    K, N = 256, 24
    layer = gen.uniform_layer(7100 + bits, K, N, bits)
    w = oracle.dequant_uniform_fp16_nk(layer.qweight, layer.scales, layer.zeros, bits, 128)
    assert w.shape == (N, K)
    wb = w.view(np.uint16)
    # codes straight from the bit string of each packed word (no oracle unpacking)
    P = 32 // bits
    for n in range(N):
        for k in range(0, K, 5):
            word = int(layer.qweight[k // P, n])
            q = (word >> (bits * (k % P))) & ((1 << bits) - 1)
            s = Fraction(float(layer.scales[k // 128, n]))
            z = Fraction(float(layer.zeros[k // 128, n]))
            assert int(wb[n, k]) == _expected_bits16(s * (q - z)), (n, k)


# ---------------------------------------------------------------------------
# LUT4


def test_lut4_fp16_double_rounding_case():
    """lut = 1.5, absmax = the fp32 just above (2/3)(1 + 9 * 2^-11).  The exact product is
    1 + 9 * 2^-11 + r with 0 < r < 2^-24: rounded once to fp16 it is 1 + 5 * 2^-10
    (0x3C05); rounded to fp32 first it is the fp16 midpoint 1 + 9 * 2^-11 between
    0x3C04 and 0x3C05, which ties to the even 0x3C04."""
    target = Fraction(2, 3) * (1 + Fraction(9, 2048))
    a = np.float32(float(target))
    if Fraction(float(a)) < target:
        a = np.nextafter(a, np.float32(2))
    assert Fraction(float(a)) > target
    exact = Fraction(3, 2) * Fraction(float(a))
    r = exact - (1 + Fraction(9, 2048))
    assert 0 < r < Fraction(1, 2 ** 24)
    assert _expected_bits16(exact) == 0x3C05                 # single rounding would differ
    lut = np.zeros(16, dtype=np.float16)
    lut[5] = np.float16(1.5)
    codes = np.full((128, 16), 5, dtype=np.uint8)
    absmax = np.full((2, 16), a, dtype=np.float32)
    w = oracle.dequant_lut4_fp16_nk(gen.pack_nibbles(codes), lut, absmax, 64)
    assert w.shape == (16, 128)
    assert np.all(w.view(np.uint16) == 0x3C04)


def test_lut4_fp16_bruteforce():
    K, N = 256, 32
    layer = gen.lut4_layer(7201, K, N)
    w = oracle.dequant_lut4_fp16_nk(layer.qbytes, layer.lut, layer.absmax, 64)
    assert w.shape == (N, K)
    wb = w.view(np.uint16)
    for n in range(N):
        for k in range(0, K, 3):
            byte = int(layer.qbytes[k // 2, n])
            q = (byte >> 4) if k % 2 else (byte & 0xF)
            exact = Fraction(float(layer.lut[q])) * Fraction(float(layer.absmax[k // 64, n]))
            assert int(wb[n, k]) == _expected_bits16(_fp32(exact)), (n, k)


# ---------------------------------------------------------------------------
# prefill matmul


def test_prefill_one_hot_and_bruteforce():
    K, N, M = 256, 40, 3
    layer = gen.uniform_layer(7301, K, N, 4)
    w16 = oracle.dequant_uniform_fp16_nk(layer.qweight, layer.scales, layer.zeros, 4, 128)
    x = np.zeros((2, K), dtype=np.float16)
    x[0, 17] = 1
    x[1, 200] = -2
    y = oracle.prefill_matmul(x, w16)
    assert y.shape == (2, N)
    assert np.array_equal(y[0], w16[:, 17].astype(np.float64))
    assert np.array_equal(y[1], -2 * w16[:, 200].astype(np.float64))
    xr = gen.activations(7302, M, K)
    yr = oracle.prefill_matmul(xr, w16)
    for m in range(M):
        for n in range(0, N, 7):
            exact = sum(Fraction(float(xr[m, k])) * Fraction(float(w16[n, k])) for k in range(K))
            assert abs(Fraction(float(yr[m, n])) - exact) <= Fraction(1, 2 ** 40) * (1 + abs(exact))


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_prefill_close_to_exact_weight_gemv(bits):
    K, N, M = 384, 48, 4
    layer = gen.uniform_layer(7400 + bits, K, N, bits)
    x = gen.activations(7400, M, K)
    w16 = oracle.dequant_uniform_fp16_nk(layer.qweight, layer.scales, layer.zeros, bits, 128)
    y16 = oracle.prefill_matmul(x, w16)
    y = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, bits, 128)
    w = oracle.dequant_uniform(oracle.unpack_uniform(layer.qweight, bits), layer.scales,
                               layer.zeros, 128)
    bound = np.abs(x.astype(np.float64)) @ (np.abs(w) * 2.0 ** -11)
    assert np.all(np.abs(y16 - y) <= bound * (1 + 1e-9) + 1e-300)


# ---------------------------------------------------------------------------
# plausible mistakes planted in the oracle (on the CPU) fail the pins above


def _mut_lut4_single_rounding(qbytes, lut, absmax, block):
    w = oracle.dequant_lut4(oracle.unpack_lut4(qbytes), lut, absmax, block)
    return np.ascontiguousarray(w.T).astype(np.float16)


def _mut_lut4_no_transpose(qbytes, lut, absmax, block):
    w32 = oracle.dequant_lut4_fp32(oracle.unpack_lut4(qbytes), lut, absmax, block)
    return w32.astype(np.float16)


def _mut_uniform_truncate(qweight, scales, zeros, bits, group):
    w = oracle.dequant_uniform(oracle.unpack_uniform(qweight, bits), scales, zeros, group)
    w = np.clip(w.T, -65504, 65504)
    r = w.astype(np.float16).astype(np.float64)
    step_back = np.abs(r) > np.abs(w)          # round toward zero instead of to nearest
    r[step_back] = np.nextafter(r[step_back].astype(np.float16),
                                np.float16(0)).astype(np.float64)
    return r.astype(np.float16)


def _mut_prefill_untransposed(x, w16_nk):
    return x.astype(np.float64) @ w16_nk.astype(np.float64).reshape(w16_nk.shape[1], -1)


@pytest.mark.parametrize("name,mutant,pins", [
    ("dequant_lut4_fp16_nk", _mut_lut4_single_rounding, [test_lut4_fp16_double_rounding_case]),
    ("dequant_lut4_fp16_nk", _mut_lut4_no_transpose, [test_lut4_fp16_bruteforce]),
    ("dequant_uniform_fp16_nk", _mut_uniform_truncate, [test_uniform_fp16_hand_worked_bits]),
    ("prefill_matmul", _mut_prefill_untransposed, [test_prefill_one_hot_and_bruteforce]),
])
def test_mutants_fail_pins(monkeypatch, name, mutant, pins):
    monkeypatch.setattr(oracle, name, mutant)
    for pin in pins:
        with pytest.raises((AssertionError, ValueError, IndexError)):
            pin()
