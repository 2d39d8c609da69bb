"""Group sizes 64 and 32 (finer groups, parameters per sub-group) and per-channel
quantization (group = K) on the GPU, against the fp64 oracle at the same group size,
through the C ABI: W2 / W4 / W8, M from 1 to 16, shapes with ragged tile and block tails,
capped grids that exercise the split-K fix-up, and the 8192 x 28672 layer on sampled
columns."""
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


@functools.lru_cache(maxsize=16)
def _layer(seed, K, N, bits, group):
    return gen.uniform_layer(seed, K, N, bits, group=group)


def _run(lay, x):
    y = lay.forward(torch.from_numpy(x).to(DEV))
    torch.cuda.synchronize()
    assert lay.read_error() == 0, "a device wait gave up"
    return y.float().cpu().numpy()


@pytest.mark.parametrize("M", [1, 3, 8, 9, 16])
@pytest.mark.parametrize("K,N", [(640, 208), (1024, 512)])
@pytest.mark.parametrize("group", [32, 64, "K"])
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_group_parity(bits, group, K, N, M):
    g = K if group == "K" else group
    u = _layer(1600 + bits, K, N, bits, g)
    lay = layers.from_uniform(u, DEV)
    x = gen.activations(1601 + M, M, K)
    ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, bits, g)
    assert_parity(_run(lay, x), ref, what=f"w{bits} g={g} {K}x{N} M={M}")


@pytest.mark.parametrize("cap", ["1", "7", "29"])
@pytest.mark.parametrize("group", [32, 64])
@pytest.mark.parametrize("M", [1, 5, 12])
def test_group_split_k_fixup(group, M, cap):
    K, N = 1408, 416
    old = os.environ.get("QLINEAR_MAX_CTAS")
    os.environ["QLINEAR_MAX_CTAS"] = cap
    try:
        u = _layer(1700, K, N, 4, group)
        lay = layers.from_uniform(u, DEV)
        x = gen.activations(1701 + M, M, K)
        ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 4, group)
        for _ in range(2):
            assert_parity(_run(lay, x), ref, what=f"w4 g={group} cap={cap} M={M}")
    finally:
        if old is None:
            os.environ.pop("QLINEAR_MAX_CTAS", None)
        else:
            os.environ["QLINEAR_MAX_CTAS"] = old


def test_group_one_hot_exact_and_zero():
    """x = e_k: y = s (q - z) of row k (fp32-exact), rounded once to fp16."""
    K, N = 512, 144
    for group in (32, 64):
        u = _layer(1800, K, N, 4, group)
        lay = layers.from_uniform(u, DEV)
        x = np.zeros((2, K), dtype=np.float16)
        x[0, 37] = 1
        x[1, 300] = 1
        y = lay.forward(torch.from_numpy(x).to(DEV))
        torch.cuda.synchronize()
        ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 4, group).astype(np.float16)
        assert np.array_equal(y.cpu().numpy().view(np.uint16), ref.view(np.uint16))
        z = lay.forward(torch.zeros((3, K), dtype=torch.float16, device=DEV))
        torch.cuda.synchronize()
        assert torch.all(z == 0)


@pytest.mark.slow
@pytest.mark.parametrize("group", [32, "K"])
def test_group_full_size_sampled(group):
    K, N = 8192, 28672
    g = K if group == "K" else group
    u = gen.uniform_layer(gen.workload_seed(6, 0), K, N, 4, group=g)
    lay = layers.from_uniform(u, DEV)
    x = gen.activations(1900, 1, K)
    y = _run(lay, x)
    rs = np.random.default_rng(19)
    cols = np.unique(np.concatenate([rs.choice(N, 128, replace=False),
                                     [0, 15, 16, 127, 128, N - 129, N - 16, N - 1]]))
    ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 4, g, cols=cols)
    assert_parity(y[:, cols], ref, what=f"w4 g={g} full")
