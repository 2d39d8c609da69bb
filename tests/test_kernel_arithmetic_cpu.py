"""The exactness facts the CUDA kernels are built on, checked exhaustively with IEEE fp16
arithmetic on the CPU (NumPy float16 rounds to nearest even, as the GPU's fp16 units do):

* GEMV fragments: a code field left in place by an AND mask (bit offset `shift` inside a
  16-bit half, all other bits zero) is, read as fp16, exactly code * 2^(shift - 24): a
  subnormal (or a small normal) with no rounding, so the tensor core sees the code times a
  power of two;
* stand-alone dequantization: OR-ing a field at offset sh into the mantissa of 2^(10 - sh)
  gives exactly 2^(10 - sh) + q, the subtraction of 2^(10 - sh) + z is exact, and one fp16
  multiply by s rounds the exact s (q - z) once (the oracle's fp16 value);
* W3's high-bit plane: a bit shifted to position 0 is exactly 2^-24.
"""
import numpy as np
import pytest


def _f16(bits):
    return np.array(bits, dtype=np.uint16).view(np.float16)


# (bits, shift) pairs the GEMV's masks leave: W4 0/4, W2 0/2/4/6, W8 0, W3 plane 0
FIELDS = [(4, 0), (4, 4), (2, 0), (2, 2), (2, 4), (2, 6), (8, 0), (1, 0)]


@pytest.mark.parametrize("bits,shift", FIELDS)
def test_masked_field_is_code_times_power_of_two(bits, shift):
    q = np.arange(1 << bits, dtype=np.uint32)
    v = _f16((q << shift).astype(np.uint16)).astype(np.float64)
    assert np.array_equal(v, q.astype(np.float64) * 2.0 ** (shift - 24))


@pytest.mark.parametrize("bits,shift", [(4, 0), (4, 4), (2, 0), (2, 2), (2, 4), (2, 6), (8, 0)])
def test_magic_number_difference_is_exact(bits, shift):
    magic = (25 - shift) << 10                      # fp16 bits of 2^(10 - shift)
    base = 2.0 ** (10 - shift)
    q = np.arange(1 << bits, dtype=np.uint32)
    a = _f16((magic | (q << shift)).astype(np.uint16))
    assert np.array_equal(a.astype(np.float64), base + q)
    for z in range(1 << bits):
        zb = np.float16(base + z)
        assert float(zb) == base + z                # the zero offset is exact too
        d = (a - zb).astype(np.float64)             # fp16 subtraction
        assert np.array_equal(d, q.astype(np.float64) - z)


def test_one_fp16_multiply_rounds_the_exact_product_once():
    rs = np.random.default_rng(0)
    # scales: random normal and subnormal fp16 bit patterns, plus the extremes
    s_bits = np.concatenate([rs.integers(1, 0x7BFF, size=3000), [1, 0x03FF, 0x0400, 0x7BFF]])
    s = _f16(s_bits.astype(np.uint16))
    d = np.arange(-255, 256, dtype=np.float16)      # every q - z of 8-bit codes
    with np.errstate(over="ignore"):                # large s x 255 overflows to inf on both sides
        prod16 = (d[None, :] * s[:, None])          # fp16 x fp16 -> fp16, rounded once
        exact = (d.astype(np.float64)[None, :] * s.astype(np.float64)[:, None]).astype(np.float16)
    assert np.array_equal(prod16.view(np.uint16), exact.view(np.uint16))
