"""Pins of the fp64 oracle against facts that do not come from the oracle.

* bounds against the unquantized fp32 weights (min-max rounding error is at
  most half a step), which fail on a dropped term, a wrong sign or index or a
  transposed operand;
* the exact-integer form of the deferred-dequantization identity (QFactory
  page, observation 2): eager and deferred group sums agree bit for bit;
* brute force with exact rationals on tiny inputs, unpacking from bit strings;
* special cases: x = 0, one-hot x, all codes equal to the zero point,
  linearity in x.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from synth import gen


def _bound_uniform(layer, w):
    """Per-element bound on |w - s (q - z)| from the min-max recipe."""
    s = layer.scales.astype(np.float64)
    s32 = layer.scales32.astype(np.float64)
    slack = s / 2 + ((1 << layer.bits) - 1) * np.abs(s - s32)
    gidx = np.arange(layer.K) // layer.group
    return slack[gidx, :]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_quantizer_invariants(bits):
    K, N = 512, 96
    layer = gen.uniform_layer(11, K, N, bits)
    w = gen.weights(11, K, N).astype(np.float64)
    codes = oracle.unpack_uniform(layer.qweight, bits)
    qmax = (1 << bits) - 1
    assert codes.max() <= qmax
    z = layer.zeros.astype(np.float64)
    assert z.min() >= 0 and z.max() <= qmax and np.array_equal(z, np.rint(z))
    deq = oracle.dequant_uniform(codes, layer.scales, layer.zeros, layer.group)
    err = np.abs(w - deq)
    assert np.all(err <= _bound_uniform(layer, w) * (1 + 1e-12))
    # codes not at the clamp edges are within half a (stored) step
    s = layer.scales.astype(np.float64)[np.arange(K) // 128, :]
    inner = (codes > 0) & (codes < qmax)
    assert np.all(err[inner] <= s[inner] / 2 * (1 + 1e-12))
    # the group minimum maps to code 0 (rint is odd-symmetric)
    wg = w.reshape(K // 128, 128, N)
    cg = codes.reshape(K // 128, 128, N)
    amin = wg.argmin(axis=1)
    assert np.all(np.take_along_axis(cg, amin[:, None, :], axis=1) == 0)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_unpack_matches_bitstring_bruteforce(bits):
    rs = np.random.default_rng(5)
    K, N = 64, 3
    words = rs.integers(0, 2 ** 32, size=(K * bits // 32, N), dtype=np.uint64).astype(np.uint32)
    codes = oracle.unpack_uniform(words, bits)
    assert codes.shape == (K, N)
    for n in range(N):
        # the column's bit stream, bit 0 of word 0 first
        stream = "".join(format(int(words[j, n]), "032b")[::-1] for j in range(words.shape[0]))
        for k in range(K):
            field = stream[bits * k: bits * k + bits][::-1]
            assert codes[k, n] == int(field, 2)
    # and packing the unpacked codes gives the words back
    assert np.array_equal(gen.pack_codes(codes, bits), words)


def test_w3_hand_worked_words():
    """Codes 0..7 repeating: the stream 000 001 010 011 100 101 110 111 ... (each field written
    least-significant bit first) packs 32 codes into three words; the first word holds codes
    0..9 and the low two bits of code 10 (= 2), i.e. 0b10_001_000_111_110_101_100_011_010_001_000
    read from bit 31 down."""
    codes = (np.arange(32) % 8).astype(np.uint8)[:, None]
    w = gen.pack_codes(codes, 3)
    assert w.shape == (3, 1)
    assert int(w[0, 0]) == 0b10001000111110101100011010001000
    assert np.array_equal(oracle.unpack_uniform(w, 3)[:, 0], codes[:, 0])


def test_unpack_lut4_bruteforce():
    rs = np.random.default_rng(6)
    b = rs.integers(0, 256, size=(10, 4), dtype=np.uint8)
    codes = oracle.unpack_lut4(b)
    for j in range(10):
        for n in range(4):
            assert codes[2 * j, n] == int(b[j, n]) % 16
            assert codes[2 * j + 1, n] == int(b[j, n]) // 16
    assert np.array_equal(gen.pack_nibbles(codes), b)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("M", [1, 3, 16])
def test_gemv_within_quantization_bound_of_unquantized(bits, M):
    K, N = 640, 64
    layer = gen.uniform_layer(21, K, N, bits)
    w = gen.weights(21, K, N).astype(np.float64)
    x = gen.activations(21, M, K)
    y = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, bits, 128)
    y_unq = x.astype(np.float64) @ w
    bound = np.abs(x.astype(np.float64)) @ _bound_uniform(layer, w)
    assert np.all(np.abs(y - y_unq) <= bound * (1 + 1e-9) + 1e-12)
    # the bound is not vacuous: the error shrinks with the bit width as min-max predicts
    # (step = range / (2^b - 1), uniform rounding error of rms step / sqrt(12))
    ratio = np.linalg.norm(y - y_unq) / np.linalg.norm(y_unq)
    assert ratio < {2: 0.7, 3: 0.35, 4: 0.15, 8: 0.01}[bits]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_eager_equals_deferred_exact_integers(bits):
    K, N, M = 384, 40, 5
    layer = gen.uniform_layer(31, K, N, bits)
    x = gen.activations(31, M, K)
    x[0, :7] = np.float16(6.1e-5) * np.arange(7)  # subnormal and tiny fp16 values
    codes = oracle.unpack_uniform(layer.qweight, bits)
    E = oracle.eager_group_sums(x, codes, layer.zeros, 128)
    D = oracle.deferred_group_sums(x, codes, layer.zeros, 128)
    assert np.array_equal(E, D)
    y_def = oracle.gemv_from_group_sums(D, layer.scales)
    y = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, bits, 128)
    assert np.allclose(y_def, y, rtol=1e-12, atol=1e-12)


def _fraction_gemv(x, words, scales, zeros, bits, group):
    """Exact rational y from bit strings (independent of NumPy unpacking)."""
    M, K = x.shape
    N = words.shape[1]
    y = [[Fraction(0)] * N for _ in range(M)]
    for n in range(N):
        # the column's little-endian bit stream, code k at bits [bits*k, bits*k + bits)
        stream = "".join(format(int(words[j, n]), "032b")[::-1] for j in range(words.shape[0]))
        col = [int(stream[bits * k: bits * (k + 1)][::-1], 2) for k in range(K)]
        for m in range(M):
            acc = Fraction(0)
            for k in range(K):
                g = k // group
                acc += Fraction(float(x[m, k])) * Fraction(float(scales[g, n])) * (col[k] - int(zeros[g, n]))
            y[m][n] = acc
    return y


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_tiny_bruteforce_fractions(bits):
    for (K, N, M) in [(128, 8, 1), (256, 3, 2), (512, 2, 16)]:
        layer = gen.uniform_layer(41 + K, K, N, bits)
        x = gen.activations(41 + K, M, K)
        y = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, bits, 128)
        yf = _fraction_gemv(x, layer.qweight, layer.scales, layer.zeros, bits, 128)
        for m in range(M):
            for n in range(N):
                exact = float(yf[m][n])
                assert abs(y[m, n] - exact) <= 1e-15 * max(1.0, abs(exact)) * K


def test_special_cases():
    K, N = 256, 24
    layer = gen.uniform_layer(51, K, N, 4)
    w = gen.weights(51, K, N).astype(np.float64)
    x0 = np.zeros((2, K), dtype=np.float16)
    y0 = oracle.gemv_uniform(x0, layer.qweight, layer.scales, layer.zeros, 4, 128)
    assert np.all(y0 == 0)
    # one-hot x reproduces one dequantized row, which is within the rounding bound of W
    kk = 133
    x1 = np.zeros((1, K), dtype=np.float16)
    x1[0, kk] = 1
    y1 = oracle.gemv_uniform(x1, layer.qweight, layer.scales, layer.zeros, 4, 128)[0]
    assert np.all(np.abs(y1 - w[kk]) <= _bound_uniform(layer, w)[kk] * (1 + 1e-12))
    # all codes equal to the zero point -> y = 0 for any x
    zcodes = np.repeat(layer.zeros.astype(np.uint8), 128, axis=0)
    qz = gen.pack_codes(zcodes, 4)
    xr = gen.activations(51, 3, K)
    assert np.all(oracle.gemv_uniform(xr, qz, layer.scales, layer.zeros, 4, 128) == 0)
    # linearity in x
    xa = gen.activations(52, 2, K)
    xb = gen.activations(53, 2, K)
    ya = oracle.gemv_uniform(xa, layer.qweight, layer.scales, layer.zeros, 4, 128)
    yb = oracle.gemv_uniform(xb, layer.qweight, layer.scales, layer.zeros, 4, 128)
    xab = np.concatenate([xa, xb], axis=0)
    yab = oracle.gemv_uniform(xab, layer.qweight, layer.scales, layer.zeros, 4, 128)
    assert np.allclose(yab, np.concatenate([ya, yb]), rtol=0, atol=1e-13)


def test_column_subset_matches_full():
    K, N = 256, 40
    layer = gen.uniform_layer(61, K, N, 4)
    x = gen.activations(61, 3, K)
    y = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, 4, 128)
    cols = [0, 7, 39, 12]
    ys = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, 4, 128, cols=cols)
    assert np.array_equal(ys, y[:, cols])


# ---------------------------------------------------------------------------
# LUT4


def test_lut_table_recipe():
    lut = gen.lut16(3003)
    v = lut.astype(np.float64)
    assert lut.dtype == np.float16 and lut.shape == (16,)
    assert np.all(np.diff(v) > 0)
    assert v[0] == -1 and v[-1] == 1 and 0.0 in v
    assert np.all(np.abs(v) <= 1)


def test_lut4_codes_nearest_and_bounds():
    K, N = 256, 48
    layer = gen.lut4_layer(3001, K, N)
    w = gen.weights(3001, K, N).astype(np.float64)
    codes = oracle.unpack_lut4(layer.qbytes)
    assert np.array_equal(codes, layer.codes)
    lut = layer.lut.astype(np.float64)
    a = layer.absmax.astype(np.float64)
    # absmax is the block maximum of |w|
    assert np.array_equal(a, np.abs(w.reshape(K // 64, 64, N)).max(axis=1))
    # brute force nearest entry on a sample, lower index on ties
    rs = np.random.default_rng(0)
    for _ in range(300):
        k, n = int(rs.integers(K)), int(rs.integers(N))
        r = w[k, n] / a[k // 64, n]
        d = [abs(r - t) for t in lut]
        best = min(range(16), key=lambda c: (d[c], c))
        assert codes[k, n] == best
    deq = oracle.dequant_lut4(codes, layer.lut, layer.absmax, 64)
    gap = np.diff(lut).max()
    bidx = np.arange(K) // 64
    assert np.all(np.abs(w - deq) <= a[bidx, :] * gap / 2 * (1 + 1e-12))
    x = gen.activations(3001, 2, K)
    y = oracle.gemv_lut4(x, layer.qbytes, layer.lut, layer.absmax, 64)
    bound = np.abs(x.astype(np.float64)) @ (a[bidx, :] * gap / 2)
    assert np.all(np.abs(y - x.astype(np.float64) @ w) <= bound * (1 + 1e-9))


def test_lut4_dequant_fp32_is_single_rounding():
    lut = gen.lut16(3002)
    a = np.array([[np.float32(0.0123)], [np.float32(3.7e-3)]], dtype=np.float32)
    codes = np.arange(16, dtype=np.uint8).repeat(8)[:128, None]
    deq32 = oracle.dequant_lut4_fp32(codes, lut, a, 64)[:, 0]
    for k in range(128):
        exact = Fraction(float(lut[codes[k, 0]])) * Fraction(float(a[k // 64, 0]))
        # fp32 round-to-nearest of the exact product
        assert Fraction(float(deq32[k])) == Fraction(float(np.float32(float(exact)))) or \
            abs(Fraction(float(deq32[k])) - exact) <= abs(Fraction(float(np.float32(float(exact)))) - exact)


# ---------------------------------------------------------------------------
# outlier Tile-COO


def test_tilecoo_structure_and_bound():
    K, N = 256, 384
    lay = gen.outlier_layer(4001, K, N)
    off = lay.tile_offsets.astype(np.int64)
    T = (K // 128) * (N // 128)
    nnz = gen.outlier_count(K, N)
    assert off.shape == (T + 1,) and off[0] == 0 and off[-1] == nnz and np.all(np.diff(off) >= 0)
    assert lay.tile_rc.max() < 128
    # entries sorted by (row, col) inside each tile, no duplicates
    for t in range(T):
        rc = lay.tile_rc[off[t]:off[t + 1]].astype(np.int64)
        key = rc[:, 0] * 128 + rc[:, 1]
        assert np.all(np.diff(key) > 0)
    dense_o = oracle.tilecoo_to_dense(lay.tile_offsets, lay.tile_rc, lay.tile_vals, K, N)
    nzk, nzn = np.nonzero(dense_o)
    flat = np.sort(nzk * N + nzn)
    # an fp16 value of 10 w can be 0 only for |w| tiny; the stored positions are the drawn ones
    assert set(flat.tolist()) <= set(lay.positions.tolist())
    # each outlier position holds the x10 weight rounded to fp16
    w = gen.weights(4001, K, N).reshape(-1)
    want = (w[lay.positions] * np.float32(10)).astype(np.float16).astype(np.float64)
    assert np.array_equal(dense_o.reshape(-1)[lay.positions], want)
    assert np.allclose(want, 10 * w[lay.positions].astype(np.float64), rtol=2 ** -11, atol=0)
    # dense slot of every outlier is the zero code
    codes = oracle.unpack_uniform(lay.dense.qweight, 4)
    k, n = lay.positions // N, lay.positions % N
    assert np.array_equal(codes[k, n], lay.dense.zeros.astype(np.uint8)[k // 128, n])
    # y against the unquantized weights (with outliers scaled) within the rounding bounds
    x = gen.activations(4001, 4, K)
    y = oracle.gemv_outlier(x, lay.dense.qweight, lay.dense.scales, lay.dense.zeros,
                            lay.tile_offsets, lay.tile_rc, lay.tile_vals, 4, 128)
    wf = lay.w_full.astype(np.float64)
    s = lay.dense.scales.astype(np.float64)
    s32 = lay.dense.scales32.astype(np.float64)
    ebound = (s / 2 + 15 * np.abs(s - s32))[np.arange(K) // 128, :]
    ebound.reshape(-1)[lay.positions] = np.abs(wf.reshape(-1)[lay.positions]) * 2.0 ** -11
    bound = np.abs(x.astype(np.float64)) @ ebound
    assert np.all(np.abs(y - x.astype(np.float64) @ wf) <= bound * (1 + 1e-9) + 1e-12)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("group", [32, 64, "K"])
def test_finer_and_per_channel_groups_within_bound(bits, group):
    """Groups of 32 and 64 and per-channel (one group of K): the element-wise min-max bound
    and the layer bound hold with the group's own scales, so a group index taken at the
    wrong granularity (for example k // 128) fails."""
    K, N, M = 256, 24, 3
    g = K if group == "K" else group
    layer = gen.uniform_layer(81 + bits, K, N, bits, group=g)
    assert layer.scales.shape == (K // g, N)
    w = gen.weights(81 + bits, K, N).astype(np.float64)
    deq = oracle.dequant_uniform(oracle.unpack_uniform(layer.qweight, bits), layer.scales,
                                 layer.zeros, g)
    el = _bound_uniform(layer, w)
    assert np.all(np.abs(deq - w) <= el * (1 + 1e-12))
    x = gen.activations(81, M, K)
    y = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, bits, g)
    bound = np.abs(x.astype(np.float64)) @ el
    assert np.all(np.abs(y - x.astype(np.float64) @ w) <= bound * (1 + 1e-9) + 1e-12)
    if g < 128:  # the finer scales really differ inside a 128-element span
        assert not np.array_equal(layer.scales[0], layer.scales[1])
