"""Hand-derived worked examples pin the quantizer recipe and the oracle.

The pages print no numeric example, so each fixture under ``tests/golden``
builds one from dyadic weights whose scale, zero, codes, packed words and
outputs follow by hand from the definitions (derivations inside each file,
with the passage they follow).
"""
import numpy as np

import oracle
from synth import gen


def _x_rows(kinds, K):
    rows = []
    for kind in kinds:
        if kind == "ones":
            rows.append(np.ones(K))
        elif kind == "alternating":
            rows.append((-1.0) ** np.arange(K))
        else:
            raise ValueError(kind)
    return np.array(rows, dtype=np.float16)


def test_w4_handworked(golden):
    g = golden("w4_handworked.json")
    K, N = g["K"], g["N"]
    k = np.arange(K)
    w = np.stack([((k % 16) - 5) / 64.0, (k % 16) / 32.0 - 0.25], axis=1).astype(np.float32)
    layer = gen.uniform_layer(0, K, N, bits=4, w=w)
    assert np.array_equal(layer.scales.astype(np.float64), np.array(g["scales"]))
    assert np.array_equal(layer.zeros.astype(np.float64), np.array(g["zeros"], dtype=np.float64))
    assert np.array_equal(layer.codes[:, 0], k % 16) and np.array_equal(layer.codes[:, 1], k % 16)
    assert np.all(layer.qweight[0::2] == g["qweight_even_word"])
    assert np.all(layer.qweight[1::2] == g["qweight_odd_word"])
    codes = oracle.unpack_uniform(layer.qweight, 4)
    assert np.array_equal(codes, layer.codes)
    x = _x_rows(g["x_rows"], K)
    y = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, 4, 128)
    assert np.array_equal(y, np.array(g["y"]))


def test_w2_handworked(golden):
    g = golden("w2_handworked.json")
    K = g["K"]
    k = np.arange(K)
    w = (((k % 4) - 1) / 8.0).astype(np.float32)[:, None]
    layer = gen.uniform_layer(0, K, 1, bits=2, w=w)
    assert float(layer.scales[0, 0]) == g["scales"][0][0]
    assert float(layer.zeros[0, 0]) == g["zeros"][0][0]
    assert np.all(layer.qweight == g["qweight_word"])
    x = _x_rows(g["x_rows"], K)
    y = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, 2, 128)
    assert np.array_equal(y, np.array(g["y"]))


def test_w8_handworked(golden):
    g = golden("w8_handworked.json")
    K = g["K"]
    k = np.arange(K)
    w = ((2 * k - 100) / 1024.0)
    w[127] = 155 / 1024.0
    layer = gen.uniform_layer(0, K, 1, bits=8, w=w.astype(np.float32)[:, None])
    assert float(layer.scales[0, 0]) == g["scales"][0][0]
    assert float(layer.zeros[0, 0]) == g["zeros"][0][0]
    assert int(layer.qweight[0, 0]) == g["qweight_word0"]
    codes = oracle.unpack_uniform(layer.qweight, 8)[:, 0]
    assert np.array_equal(codes[:127], 2 * k[:127]) and codes[127] == 255
    x = _x_rows(g["x_rows"], K)
    y = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, 8, 128)
    assert np.array_equal(y, np.array(g["y"]))


def test_lut4_handworked(golden):
    g = golden("lut4_handworked.json")
    K = g["K"]
    lut = np.array(g["lut"], dtype=np.float16)
    w = np.zeros(K, dtype=np.float32)
    w[:64] = lut.astype(np.float32)[np.arange(64) % 16] / 2
    w[64] = -0.3125
    w[65] = 0.5
    layer = gen.lut4_layer(0, K, 1, w=w[:, None], lut=lut)
    assert np.array_equal(layer.absmax, np.array(g["absmax"], dtype=np.float32))
    assert list(layer.qbytes[:32, 0]) == g["bytes_block0"] * 4
    codes = oracle.unpack_lut4(layer.qbytes)[:, 0]
    assert np.array_equal(codes[:64], np.arange(64) % 16)
    assert list(codes[64:66]) == g["codes_block1_first_two"]
    assert np.all(codes[66:128] == g["zero_code"]) and np.all(codes[128:] == g["zero_code"])
    x = np.zeros((1, K), dtype=np.float16)
    x[0, :64] = 1
    y = oracle.gemv_lut4(x, layer.qbytes, lut, layer.absmax, 64)
    assert y[0, 0] == g["y_ones_block0_only"]
    # the fp32 dequantized value of entry +-1 is exactly +-absmax, of entry 0 exactly 0
    deq = oracle.dequant_lut4_fp32(codes[:, None], lut, layer.absmax, 64)[:, 0]
    assert deq[15] == np.float32(0.5) and deq[0] == np.float32(-0.5) and deq[7] == 0


def test_tilecoo_handworked(golden):
    g = golden("tilecoo_handworked.json")
    K, N = g["K"], g["N"]
    codes = np.full((K, N), 8, dtype=np.uint8)
    qweight = gen.pack_codes(codes, 4)
    scales = np.full((1, N), 1 / 16, dtype=np.float16)
    zeros = np.full((1, N), 8, dtype=np.float16)
    offsets = np.array(g["offsets"], dtype=np.uint32)
    rc = np.array(g["rc"], dtype=np.uint8)
    vals = np.array(g["vals"], dtype=np.float16)
    x1 = np.ones((1, K), dtype=np.float16)
    xr = (np.arange(K) / 128.0).astype(np.float16)[None, :]
    for x, exp in ((x1, g["y_ones"]), (xr, g["y_ramp"])):
        y = oracle.gemv_outlier(x, qweight, scales, zeros, offsets, rc, vals, 4, 128)
        want = np.zeros(N)
        for c, v in exp.items():
            want[int(c)] = v
        assert np.array_equal(y[0], want)
