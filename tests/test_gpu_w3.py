"""3-bit codes (two bit planes) on the GPU, through the C ABI, against the fp64 oracle:
the debug decode bit-exact, GEMV parity for M = 1..16 on shapes with ragged tile and block
tails, per-channel parameters, capped grids (split-K fix-up), one-hot x bit-exact."""
import functools
import os

import numpy as np
import pytest

import oracle
from synth import gen
from tests.helpers import assert_parity

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from weight_only_quantized_gemv_b200 import layers

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


@functools.lru_cache(maxsize=8)
def _layer(seed, K, N, group=128):
    return gen.uniform_layer(seed, K, N, 3, group=group)


def _run(lay, x):
    y = lay.forward(torch.from_numpy(x).to(DEV))
    torch.cuda.synchronize()
    assert lay.read_error() == 0, "a device wait gave up"
    return y.float().cpu().numpy()


@pytest.mark.parametrize("K,N", [(256, 48), (640, 208)])
def test_w3_debug_decode_bit_exact(K, N):
    u = _layer(2000, K, N)
    lay = layers.from_uniform(u, DEV)
    codes = lay.debug_unpack().cpu().numpy()
    assert np.array_equal(codes, oracle.unpack_uniform(u.qweight, 3))
    w = lay.debug_dequant().cpu().numpy()
    ref = oracle.dequant_uniform(oracle.unpack_uniform(u.qweight, 3), u.scales, u.zeros, 128)
    assert np.array_equal(w, ref.astype(np.float32))


@pytest.mark.parametrize("M", [1, 2, 5, 8, 9, 16])
@pytest.mark.parametrize("K,N", [(128, 16), (640, 208), (1024, 512), (2048, 1152)])
def test_w3_parity(K, N, M):
    u = _layer(2001, K, N)
    x = gen.activations(2002 + M, M, K)
    ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 3, 128)
    assert_parity(_run(layers.from_uniform(u, DEV), x), ref, what=f"w3 {K}x{N} M={M}")


@pytest.mark.parametrize("M", [1, 12])
def test_w3_per_channel(M):
    K, N = 1024, 208
    u = _layer(2003, K, N, group=K)
    x = gen.activations(2004 + M, M, K)
    ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 3, K)
    assert_parity(_run(layers.from_uniform(u, DEV), x), ref, what=f"w3 per-channel M={M}")


@pytest.mark.parametrize("cap", ["1", "7", "29"])
@pytest.mark.parametrize("M", [1, 6, 13])
def test_w3_split_k_fixup(M, cap):
    K, N = 1408, 416
    old = os.environ.get("QLINEAR_MAX_CTAS")
    os.environ["QLINEAR_MAX_CTAS"] = cap
    try:
        u = _layer(2005, K, N)
        x = gen.activations(2006 + M, M, K)
        ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 3, 128)
        lay = layers.from_uniform(u, DEV)
        for _ in range(2):
            assert_parity(_run(lay, x), ref, what=f"w3 cap={cap} M={M}")
    finally:
        if old is None:
            os.environ.pop("QLINEAR_MAX_CTAS", None)
        else:
            os.environ["QLINEAR_MAX_CTAS"] = old


def test_w3_one_hot_bit_exact():
    K, N = 512, 144
    u = _layer(2007, K, N)
    lay = layers.from_uniform(u, DEV)
    x = np.zeros((3, K), dtype=np.float16)
    for m, k in enumerate((5, 200, 511)):
        x[m, k] = 1
    y = lay.forward(torch.from_numpy(x).to(DEV))
    torch.cuda.synchronize()
    ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 3, 128).astype(np.float16)
    assert np.array_equal(y.cpu().numpy().view(np.uint16), ref.view(np.uint16))
