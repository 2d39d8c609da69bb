"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch them.

Each mutant replaces one oracle function for the duration of a test; the
pins used are the element-wise dequantization bound and the bound of the
layer output against the unquantized weights, plus the hand-derived W4
golden example.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import qlinear_oracle as qo
from synth import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "w4_handworked.json")


def _pins_hold(bits=4):
    K, N, M = 384, 48, 3
    layer = gen.uniform_layer(77, K, N, bits)
    w = gen.weights(77, K, N).astype(np.float64)
    x = gen.activations(77, M, K)
    y = oracle.gemv_uniform(x, layer.qweight, layer.scales, layer.zeros, bits, 128)
    s = layer.scales.astype(np.float64)
    s32 = layer.scales32.astype(np.float64)
    el = (s / 2 + ((1 << bits) - 1) * np.abs(s - s32))[np.arange(K) // 128, :]
    bound = np.abs(x.astype(np.float64)) @ el
    ok_bound = bool(np.all(np.abs(y - x.astype(np.float64) @ w) <= bound * (1 + 1e-9) + 1e-12))
    deq = oracle.dequant_uniform(oracle.unpack_uniform(layer.qweight, bits), layer.scales,
                                 layer.zeros, 128)
    ok_bound = ok_bound and bool(np.all(np.abs(w - deq) <= el * (1 + 1e-12)))
    with open(GOLDEN) as f:
        g = json.load(f)
    k = np.arange(128)
    wg = np.stack([((k % 16) - 5) / 64.0, (k % 16) / 32.0 - 0.25], axis=1).astype(np.float32)
    lay = gen.uniform_layer(0, 128, 2, bits=4, w=wg)
    xg = np.stack([np.ones(128), (-1.0) ** k]).astype(np.float16)
    yg = oracle.gemv_uniform(xg, lay.qweight, lay.scales, lay.zeros, 4, 128)
    ok_golden = bool(np.array_equal(yg, np.array(g["y"])))
    return ok_bound and ok_golden


def test_unmutated_pins_hold():
    assert _pins_hold()


def _mut_zero_sign(codes, scales, zeros, group, cols=None):
    s = qo._col_select(scales, cols).astype(np.float64)
    z = qo._col_select(zeros, cols).astype(np.float64)
    gidx = np.arange(codes.shape[0]) // group
    return s[gidx, :] * (codes.astype(np.float64) + z[gidx, :])


def _mut_drop_zero(codes, scales, zeros, group, cols=None):
    s = qo._col_select(scales, cols).astype(np.float64)
    gidx = np.arange(codes.shape[0]) // group
    return s[gidx, :] * codes.astype(np.float64)


def _mut_group_index(codes, scales, zeros, group, cols=None):
    s = qo._col_select(scales, cols).astype(np.float64)
    z = qo._col_select(zeros, cols).astype(np.float64)
    G = s.shape[0]
    gidx = np.arange(codes.shape[0]) % G  # wrong: interleaved instead of contiguous groups
    return s[gidx, :] * (codes.astype(np.float64) - z[gidx, :])


def _mut_bit_order(qweight, bits, cols=None):
    words = qo._col_select(qweight, cols).astype(np.uint32)
    P = 32 // bits
    mask = np.uint32((1 << bits) - 1)
    codes = np.empty((words.shape[0] * P, words.shape[1]), dtype=np.uint8)
    for i in range(P):  # wrong: most significant field first
        codes[i::P, :] = (words >> np.uint32(bits * (P - 1 - i))) & mask
    return codes


def _mut_transpose(x, qweight, scales, zeros, bits, group, cols=None):
    codes = qo.unpack_uniform(qweight, bits, cols)
    w = qo.dequant_uniform(codes, scales, zeros, group, cols)
    K, N = w.shape
    wt = w.reshape(N, K).T if K != N else w.T  # wrong: operand read transposed
    return x.astype(np.float64) @ wt


@pytest.mark.parametrize("name,target,mutant", [
    ("zero sign", "dequant_uniform", _mut_zero_sign),
    ("dropped zero term", "dequant_uniform", _mut_drop_zero),
    ("group index", "dequant_uniform", _mut_group_index),
    ("bit order", "unpack_uniform", _mut_bit_order),
    ("transposed operand", "gemv_uniform", _mut_transpose),
])
def test_planted_mistake_is_caught(monkeypatch, name, target, mutant):
    monkeypatch.setattr(qo, target, mutant)
    monkeypatch.setattr(oracle, target, mutant)
    assert not _pins_hold(), name
