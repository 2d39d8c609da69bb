"""The tensor-core prefill GEMM (tcgen05) on the GPU, through the C ABI, against the fp64
oracle on the oracle's fp16 weights.

* qlinear_prefill_fused (weights dequantized inside the GEMM) for every format, on shapes
  with a ragged last 128-row tile (N % 128 != 0) and batch sizes on both sides of the token
  tiles (128 and 256 rows of x), including a partial last token tile, with the stream-K
  schedule (tiles split between CTAs, down to one k-block per CTA on small layers) and with
  whole tiles per CTA;
* qlinear_prefill (stand-alone dequantization, then the same GEMM on the fp16 weights) at
  the batch sizes the older tests do not reach;
* the same call twice (the persistent CTAs' pipeline phases carry over between tiles, not
  between calls), and the kernels' wait flags read back as 0;
* forty calls on a layer whose CTAs each run 64 k-blocks, all bit-identical;
* one-hot rows of x: y equals the fp16 weight column bit for bit (a single exact product);
* the target layer (8192 x 28672, W4) at M = 512 on sampled columns;
* both tile forms: one CTA per 128-row tile, and a cluster pair of CTAs per 256-row tile
  (tcgen05 cta_group::2; QLINEAR_TC_PAIR selects), including layers whose last pair has
  no rows for its second CTA (N / 128 odd).
"""
import functools

import numpy as np
import pytest

import oracle
from synth import gen
from tests.helpers import assert_parity, lut4_layer, uniform_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import weight_only_quantized_gemv_b200 as ql
    from weight_only_quantized_gemv_b200 import layers

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert ql.qlinear_prefill_read_error() == 0, "a prefill kernel wait ran out"


@pytest.fixture(params=["pair", "single"])
def tile_form(request, monkeypatch):
    monkeypatch.setenv("QLINEAR_TC_PAIR", "1" if request.param == "pair" else "0")
    return request.param


def _layer(fmt, K, N, seed):
    if fmt == "lut4":
        lt = lut4_layer(seed, K, N)
        return layers.from_lut4(lt, DEV), oracle.dequant_lut4_fp16_nk(lt.qbytes, lt.lut,
                                                                      lt.absmax, 64)
    bits = int(fmt[1:])
    u = uniform_layer(seed + bits, K, N, bits)
    return layers.from_uniform(u, DEV), oracle.dequant_uniform_fp16_nk(
        u.qweight, u.scales, u.zeros, bits, 128)


def _np(t):
    torch.cuda.synchronize()
    return t.float().cpu().numpy()


@pytest.mark.parametrize("M", [1, 16, 17, 128, 129, 256, 300])
@pytest.mark.parametrize("K,N", [(384, 208), (1024, 384), (1024, 512), (2048, 1168)])
@pytest.mark.parametrize("fmt", ["w2", "w4", "w8", "lut4"])
def test_prefill_fused_parity(fmt, K, N, M, tile_form):
    lay, w16 = _layer(fmt, K, N, 700)
    x = gen.activations(1900 + M, M, K)
    y = _np(lay.prefill_fused(torch.from_numpy(x).to(DEV)))
    assert_parity(y, oracle.prefill_matmul(x, w16), what=f"fused {fmt} {K}x{N} M={M}")


@pytest.mark.parametrize("M", [1, 17, 129, 300])
@pytest.mark.parametrize("K,N", [(384, 208), (1024, 384), (2048, 1168)])
@pytest.mark.parametrize("fmt", ["w2", "w4", "lut4"])
def test_prefill_fused_whole_tiles_parity(fmt, K, N, M, tile_form):
    lay, w16 = _layer(fmt, K, N, 710)
    x = gen.activations(1930 + M, M, K)
    y = _np(lay.prefill_fused(torch.from_numpy(x).to(DEV), stream_k=False))
    assert_parity(y, oracle.prefill_matmul(x, w16), what=f"whole tiles {fmt} {K}x{N} M={M}")


def test_prefill_fused_stream_k_matches_whole_tiles(tile_form):
    """Same fp16 weights and x: the two schedules differ only in how k-blocks are summed."""
    K, N, M = 4096, 1168, 300
    lay, w16 = _layer("w4", K, N, 715)
    x = torch.from_numpy(gen.activations(1940, M, K)).to(DEV)
    a = _np(lay.prefill_fused(x, stream_k=True))
    b = _np(lay.prefill_fused(x, stream_k=False))
    assert_parity(a, b, what="stream-K vs whole tiles")
    assert_parity(a, oracle.prefill_matmul(x.cpu().numpy(), w16), what="stream-K")


def test_prefill_fused_workspace_checks():
    K, N, M = 1024, 512, 300
    lay, _ = _layer("w4", K, N, 716)
    x = torch.from_numpy(gen.activations(1941, M, K)).to(DEV)
    y = torch.empty((M, N), dtype=torch.float16, device=DEV)
    small = torch.zeros(64, dtype=torch.int32, device=DEV)
    with pytest.raises(ql.QLinearError) as err:
        ql.qlinear_prefill_fused(4, x.view(torch.int16), lay.qweight, lay.p0, lay.p1,
                                 y.view(torch.int16), M, N, K, small)
    assert err.value.status == 5  # QL_ERR_WORKSPACE
    assert ql.qlinear_prefill_workspace_bytes(M, N, K) > 0
    assert ql.qlinear_prefill_workspace_bytes(M, N + 1, K) == 0


@pytest.mark.parametrize("M", [129, 256, 300, 520])
@pytest.mark.parametrize("N", [1168, 384])
@pytest.mark.parametrize("fmt", ["w4", "lut4"])
def test_prefill_dense_tc_parity(fmt, N, M, tile_form):
    K = 1024
    lay, w16 = _layer(fmt, K, N, 720)
    x = gen.activations(1950 + M, M, K)
    wbuf = torch.empty((N, K), dtype=torch.float16, device=DEV)
    y = _np(lay.prefill(torch.from_numpy(x).to(DEV), w_fp16=wbuf))
    assert np.array_equal(wbuf.view(torch.int16).cpu().numpy().view(np.uint16),
                          w16.view(np.uint16))
    assert_parity(y, oracle.prefill_matmul(x, w16), what=f"dense tc {fmt} M={M}")


def test_prefill_fused_repeat_and_explicit_stream(tile_form):
    K, N, M = 2048, 1168, 300
    lay, w16 = _layer("w4", K, N, 730)
    x = torch.from_numpy(gen.activations(1990, M, K)).to(DEV)
    s = torch.cuda.Stream()
    ys = []
    for _ in range(3):
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device=DEV)
        with torch.cuda.stream(s):
            lay.prefill_fused(x, y, stream=s)
        s.synchronize()
        ys.append(y.view(torch.int16).cpu().numpy())
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[0], ys[2])  # deterministic
    assert_parity(ys[0].view(np.float16).astype(np.float64),
                  oracle.prefill_matmul(x.cpu().numpy(), w16), what="repeat")


@pytest.mark.parametrize("stream_k", [False, True])
@pytest.mark.parametrize("fmt", ["w2", "w4"])
def test_prefill_fused_repeat_many(fmt, stream_k, tile_form):
    """Long per-CTA runs (whole tiles: 64 k-blocks per CTA, so every ring wraps many times),
    repeated: each result bit-identical to the first, the first within tolerance.  A shared-
    memory slot released too early shows up here as results that differ between calls."""
    K, N, M = 4096, 1168, 300
    lay, w16 = _layer(fmt, K, N, 760)
    x = torch.from_numpy(gen.activations(1995, M, K)).to(DEV)
    y = torch.empty((M, N), dtype=torch.float16, device=DEV)
    first = None
    for _ in range(40):
        lay.prefill_fused(x, y, stream_k=stream_k)
        torch.cuda.synchronize()
        h = y.view(torch.int16).cpu().numpy()
        if first is None:
            first = h.copy()
            assert_parity(h.view(np.float16).astype(np.float64),
                          oracle.prefill_matmul(x.cpu().numpy(), w16), what=f"repeat {fmt}")
        else:
            assert np.array_equal(h, first)


@pytest.mark.parametrize("fmt", ["w4", "w8", "lut4"])
def test_prefill_fused_one_hot_bit_exact(fmt, tile_form):
    K, N = 1024, 400
    lay, w16 = _layer(fmt, K, N, 740)
    ks = [0, 5, 63, 64, 127, 128, 511, 1023]
    x = np.zeros((len(ks), K), dtype=np.float16)
    for m, k in enumerate(ks):
        x[m, k] = 1
    y = lay.prefill_fused(torch.from_numpy(x).to(DEV))
    torch.cuda.synchronize()
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    want = np.ascontiguousarray(w16[:, ks].T).view(np.uint16)
    assert np.array_equal(got, want)


@functools.lru_cache(maxsize=1)
def _big():
    return gen.uniform_layer(gen.workload_seed(1, 4), 8192, 28672, 4)


@pytest.mark.slow
def test_prefill_fused_full_size_sampled(tile_form):
    u = _big()
    K, N, M = u.K, u.N, 512
    rs = np.random.default_rng(7)
    cols = np.unique(np.concatenate([rs.choice(N, 96, replace=False),
                                     [0, 15, 16, 127, 128, N - 129, N - 16, N - 1]]))
    lay = layers.from_uniform(u, DEV)
    x = gen.activations(4343, M, K)
    y = _np(lay.prefill_fused(torch.from_numpy(x).to(DEV)))
    ref16 = oracle.dequant_uniform_fp16_nk(u.qweight[:, cols], u.scales[:, cols],
                                           u.zeros[:, cols], 4, 128)
    assert_parity(y[:, cols], oracle.prefill_matmul(x, ref16), what=f"fused {K}x{N} M={M}")
