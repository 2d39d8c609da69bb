"""Codebook GEMV (CodeGEMM m1v4g128) against the fp64 oracle, through the C ABI.

* The Psumbook form (qlinear_codebook): M = 1..4, shapes with one or many K ranges (a ragged
  last range at M = 1), random and nearest-centroid codes, one-hot x bit-exact, determinism
  and workspace reuse, and the 8192 x 28672 layer on sampled columns.
* The tensor-core form (qlinear_codebook_tc, the GEMV kernel with codebook lookups as A
  fragments): M = 1..16 (both M buckets, the single-row kernel), ragged blocks (N % 128 != 0),
  one-hot x bit-exact, zero x, repeat determinism, and the 8192 x 28672 layer on sampled
  columns."""
import functools

import numpy as np
import pytest

import oracle
from synth import gen
from tests.helpers import assert_parity

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import weight_only_quantized_gemv_b200 as ql

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


class CbDev:
    def __init__(self, L):
        self.L, self.K, self.N = L, L.K, L.N
        self.codes = torch.from_numpy(ql.qlinear_pack_codebook(L.codes, L.N, L.K)).to(DEV)
        self.scales = torch.from_numpy(
            ql.qlinear_pack_codebook_scales(L.scales, L.N, L.K).view(np.int16)).to(DEV)
        self.cb = torch.from_numpy(np.ascontiguousarray(L.codebook).view(np.int16)).to(DEV)
        need = max(ql.qlinear_codebook_workspace_bytes(m, L.N, L.K) for m in range(1, 5))
        self.ws = torch.zeros(max(need, 256) // 4 + 64, dtype=torch.int32, device=DEV)

    def run(self, x):
        M = x.shape[0]
        xd = torch.from_numpy(x).to(DEV).view(torch.int16)
        y = torch.empty((M, self.N), dtype=torch.int16, device=DEV)
        ql.qlinear_codebook(xd, self.codes, self.scales, self.cb, y, M, self.N, self.K, self.ws)
        torch.cuda.synchronize()
        return y.cpu().numpy().view(np.float16)


def _ref(L, x, cols=None):
    return oracle.gemv_codebook(x, L.codes, L.codebook, L.scales, 4, 128, cols)


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("K,N", [(128, 32), (256, 64), (384, 96), (1024, 512), (4096, 4096)])
def test_parity_random_codes(K, N, M):
    L = gen.codebook_layer(900 + K + N, K, N)
    d = CbDev(L)
    x = gen.activations(901 + M, M, K)
    assert_parity(d.run(x), _ref(L, x), what=f"cb {K}x{N} M={M}")


@pytest.mark.parametrize("M", [1, 4])
def test_parity_nearest_centroid_codes(M):
    K, N = 640, 160
    L = gen.codebook_layer(910, K, N, w=gen.weights(910, K, N))
    x = gen.activations(911, M, K)
    assert_parity(CbDev(L).run(x), _ref(L, x), what=f"cb nearest M={M}")


@pytest.mark.parametrize("M", [1, 3])
def test_one_hot_bit_exact_and_zero(M):
    K, N = 768, 256
    L = gen.codebook_layer(920, K, N)
    d = CbDev(L)
    x = np.zeros((M, K), dtype=np.float16)
    for m in range(M):
        x[m, 97 + 211 * m] = 1
    y = d.run(x)
    assert np.array_equal(y.view(np.uint16), _ref(L, x).astype(np.float16).view(np.uint16))
    assert np.all(d.run(np.zeros((M, K), dtype=np.float16)) == 0)


def test_deterministic_and_workspace_reuse():
    K, N = 2048, 1024
    L = gen.codebook_layer(930, K, N)
    d = CbDev(L)
    x = gen.activations(931, 2, K)
    y1 = d.run(x)
    y2 = d.run(x)
    assert np.array_equal(y1.view(np.uint16), y2.view(np.uint16))
    counters = d.ws[: N // 32].cpu().numpy()
    assert np.all(counters == 0)
    x1 = gen.activations(932, 1, K)
    assert_parity(d.run(x1), _ref(L, x1), what="after M=2")


@functools.lru_cache(maxsize=1)
def _big():
    return gen.codebook_layer(gen.workload_seed(5, 0), 8192, 28672)


@pytest.mark.slow
@pytest.mark.parametrize("M", [1, 4])
def test_full_size_sampled(M):
    L = _big()
    d = CbDev(L)
    x = gen.activations(940 + M, M, L.K)
    y = d.run(x)
    rs = np.random.default_rng(M)
    cols = np.unique(np.concatenate([rs.choice(L.N, 160, replace=False),
                                     [0, 31, 32, L.N // 2, L.N - 33, L.N - 32, L.N - 1]]))
    assert_parity(y[:, cols], _ref(L, x, cols), what=f"cb full M={M}")


# ---------------------------------------------------------------------------
# tensor-core form


class CbTcDev:
    def __init__(self, L):
        self.L, self.K, self.N = L, L.K, L.N
        self.codes = torch.from_numpy(ql.qlinear_pack_codebook_tc(L.codes, L.N, L.K)).to(DEV)
        self.scales = torch.from_numpy(
            ql.qlinear_pack_params(ql.QL_FMT_W4, np.ascontiguousarray(L.scales).view(np.uint16),
                                   L.N, L.K).view(np.int16)).to(DEV)
        self.cb = torch.from_numpy(np.ascontiguousarray(L.codebook).view(np.int16)).to(DEV)
        need = max(ql.qlinear_workspace_bytes(ql.QL_FMT_CB, m, L.N, L.K) for m in (1, 2, 9, 16))
        self.ws = torch.zeros(max(need, 256) // 4 + 64, dtype=torch.int32, device=DEV)

    def run(self, x):
        M = x.shape[0]
        xd = torch.from_numpy(x).to(DEV).view(torch.int16)
        y = torch.empty((M, self.N), dtype=torch.int16, device=DEV)
        ql.qlinear_codebook_tc(xd, self.codes, self.scales, self.cb, y, M, self.N, self.K, self.ws)
        torch.cuda.synchronize()
        assert ql.qlinear_read_error(self.ws) == 0
        return y.cpu().numpy().view(np.float16)


@pytest.mark.parametrize("M", [1, 2, 5, 8, 9, 16])
@pytest.mark.parametrize("K,N", [(128, 16), (256, 48), (1024, 208), (2048, 1168), (4096, 4096)])
def test_tc_parity_random_codes(K, N, M):
    L = gen.codebook_layer(960 + K + N, K, N)
    x = gen.activations(961 + M, M, K)
    assert_parity(CbTcDev(L).run(x), _ref(L, x), what=f"cb tc {K}x{N} M={M}")


@pytest.mark.parametrize("M", [1, 4, 16])
def test_tc_parity_nearest_centroid_codes(M):
    K, N = 640, 160
    L = gen.codebook_layer(910, K, N, w=gen.weights(910, K, N))
    x = gen.activations(911, M, K)
    assert_parity(CbTcDev(L).run(x), _ref(L, x), what=f"cb tc nearest M={M}")


@pytest.mark.parametrize("M", [1, 3, 12])
def test_tc_one_hot_bit_exact_and_zero(M):
    """A one-hot row of x picks one weight, s * C[code][k % 4]: one exact product, rounded
    once, so y equals the oracle's fp16 value bit for bit."""
    K, N = 768, 256
    L = gen.codebook_layer(970, K, N)
    d = CbTcDev(L)
    x = np.zeros((M, K), dtype=np.float16)
    for m in range(M):
        x[m, (97 + 211 * m) % K] = 1
    y = d.run(x)
    assert np.array_equal(y.view(np.uint16), _ref(L, x).astype(np.float16).view(np.uint16))
    assert np.all(d.run(np.zeros((M, K), dtype=np.float16)) == 0)


def test_tc_repeat_deterministic():
    K, N = 4096, 1168
    L = gen.codebook_layer(980, K, N)
    d = CbTcDev(L)
    x = gen.activations(981, 1, K)
    first = d.run(x)
    for _ in range(10):
        assert np.array_equal(d.run(x).view(np.uint16), first.view(np.uint16))
    assert_parity(first, _ref(L, x), what="cb tc repeat")


@pytest.mark.slow
@pytest.mark.parametrize("M", [1, 8])
def test_tc_full_size_sampled(M):
    L = _big()
    d = CbTcDev(L)
    x = gen.activations(990 + M, M, L.K)
    y = d.run(x)
    rs = np.random.default_rng(M)
    cols = np.unique(np.concatenate([rs.choice(L.N, 160, replace=False),
                                     [0, 15, 16, 127, 128, L.N - 129, L.N - 16, L.N - 1]]))
    assert_parity(y[:, cols], _ref(L, x, cols), what=f"cb tc full M={M}")


@pytest.mark.parametrize("form,M", [("tc", 1), ("tc", 16), ("psumbook", 1), ("psumbook", 4)])
def test_codebook_layer_both_forms(form, M):
    """The device layer (layers.from_codebook) runs either form on the same canonical arrays."""
    from weight_only_quantized_gemv_b200 import layers
    K, N = 1024, 512
    L = gen.codebook_layer(995, K, N)
    lay = layers.from_codebook(L, DEV)
    x = gen.activations(996 + M, M, K)
    y = lay.forward(torch.from_numpy(x).to(DEV), form=form)
    torch.cuda.synchronize()
    assert lay.read_error() == 0
    assert_parity(y.float().cpu().numpy(), _ref(L, x), what=f"cb layer {form} M={M}")
