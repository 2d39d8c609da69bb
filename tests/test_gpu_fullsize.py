"""The five workloads at their full sizes, in the launch configuration the benchmark
times, against the oracle on sampled output columns (all columns for the small one).

Columns are sampled at random plus every 128-column block boundary region that the
first and last CTAs touch, so the split-K fix-up and the first/last tiles are covered.
"""
import functools

import numpy as np
import pytest

import oracle
from synth import gen
from tests.helpers import assert_parity

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu, pytest.mark.slow]

if torch.cuda.is_available():
    from weight_only_quantized_gemv_b200 import layers

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _cols(N, seed, n=192):
    rs = np.random.default_rng(seed)
    c = set(rs.choice(N, size=min(n, N), replace=False).tolist())
    c.update([0, 1, 15, 16, 127, 128, N // 2, N - 129, N - 128, N - 17, N - 16, N - 1])
    return np.array(sorted(x for x in c if 0 <= x < N))


def _run(lay, x):
    y = lay.forward(torch.from_numpy(x).to(DEV))
    torch.cuda.synchronize()
    assert lay.read_error() == 0, "a device wait gave up"
    return y.float().cpu().numpy()


@functools.lru_cache(maxsize=1)
def _uniform(seed, K, N, bits):
    return gen.uniform_layer(seed, K, N, bits)


def test_workload0_w4_4096_all_outputs():
    K, N = 4096, 4096
    seed = gen.workload_seed(0, 0)
    u = _uniform(seed, K, N, 4)
    x = gen.activations(seed, 1, K)
    y = _run(layers.from_uniform(u, DEV), x)
    assert_parity(y, oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 4, 128), what="w0")


@pytest.mark.parametrize("j,shape", list(enumerate(gen.LLAMA_SHAPES)))
def test_workload1_w4_llama_layers(j, shape):
    K, N = shape
    seed = gen.workload_seed(1, j)
    u = _uniform(seed, K, N, 4)
    x = gen.activations(seed, 1, K)
    y = _run(layers.from_uniform(u, DEV), x)
    cols = _cols(N, seed)
    ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 4, 128, cols=cols)
    assert_parity(y[:, cols], ref, what=f"w1 {shape}")


@pytest.mark.parametrize("j,shape", list(enumerate(gen.LLAMA_SHAPES)))
def test_workload2_w2_llama_layers(j, shape):
    K, N = shape
    seed = gen.workload_seed(2, j)
    u = _uniform(seed, K, N, 2)
    x = gen.activations(seed, 1, K)
    y = _run(layers.from_uniform(u, DEV), x)
    cols = _cols(N, seed)
    ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 2, 128, cols=cols)
    assert_parity(y[:, cols], ref, what=f"w2 {shape}")


@pytest.mark.parametrize("j,shape", list(enumerate(gen.WORKLOADS[2]["w8_shapes"])))
def test_workload2_w8_trend_layers(j, shape):
    K, N = shape
    seed = gen.workload_seed(2, 10 + j)
    u = _uniform(seed, K, N, 8)
    x = gen.activations(seed, 1, K)
    y = _run(layers.from_uniform(u, DEV), x)
    cols = _cols(N, seed)
    ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 8, 128, cols=cols)
    assert_parity(y[:, cols], ref, what=f"w8 {shape}")


@pytest.mark.parametrize("j,shape", list(enumerate(gen.WORKLOADS[3]["shapes"])))
def test_workload3_lut4(j, shape):
    K, N = shape
    seed = gen.workload_seed(3, j)
    lt = gen.lut4_layer(seed, K, N)
    x = gen.activations(seed, 1, K)
    y = _run(layers.from_lut4(lt, DEV), x)
    cols = _cols(N, seed)
    ref = oracle.gemv_lut4(x, lt.qbytes, lt.lut, lt.absmax, 64, cols=cols)
    assert_parity(y[:, cols], ref, what=f"lut4 {shape}")


@pytest.mark.parametrize("j,shape", list(enumerate(gen.WORKLOADS[4]["shapes"])))
def test_workload4_outlier_m_sweep(j, shape):
    K, N = shape
    seed = gen.workload_seed(4, j)
    o = gen.outlier_layer(seed, K, N)
    lay = layers.from_outlier(o, DEV)
    cols = _cols(N, seed, n=96)
    for M in gen.WORKLOADS[4]["M"]:
        x = gen.activations(seed + 100 * M, M, K)
        y = _run(lay, x)
        ref = oracle.gemv_outlier(x, o.dense.qweight, o.dense.scales, o.dense.zeros,
                                  o.tile_offsets, o.tile_rc, o.tile_vals, 4, 128, cols=cols)
        assert_parity(y[:, cols], ref, what=f"outlier {shape} M={M}")
