"""Prefill path (stand-alone dequantization to fp16 + dense GEMM) against the oracle,
through the C ABI.

* qlinear_dequant_fp16: bit-exact fp16 weights for every format, shapes spanning
  several blocks with ragged last blocks, the hand-derived rounding cases (ties to
  even, overflow, subnormal scale, the LUT4 double rounding), and sampled columns of
  a full-size layer;
* qlinear_prefill: y = x W^T for M from 1 to several hundred against the fp64
  product on the oracle's fp16 weights, and at full size on sampled columns.
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
    from weight_only_quantized_gemv_b200 import layers

DEV = "cuda:0"
SHAPES = [(128, 16), (384, 208), (1024, 512), (640, 1040)]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def _bits(t):
    torch.cuda.synchronize()
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _oracle_w16(u):
    return oracle.dequant_uniform_fp16_nk(u.qweight, u.scales, u.zeros, u.bits, 128)


# ---------------------------------------------------------------------------
# dequantization, bit-exact


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_dequant_fp16_uniform_bit_exact(bits, K, N):
    u = uniform_layer(500 + bits, K, N, bits)
    lay = layers.from_uniform(u, DEV)
    w = lay.dequant_fp16()
    assert tuple(w.shape) == (N, K)
    assert np.array_equal(_bits(w), _oracle_w16(u).view(np.uint16))


@pytest.mark.parametrize("K,N", SHAPES)
def test_dequant_fp16_lut4_bit_exact(K, N):
    lt = lut4_layer(601, K, N)
    lay = layers.from_lut4(lt, DEV)
    w = lay.dequant_fp16()
    ref = oracle.dequant_lut4_fp16_nk(lt.qbytes, lt.lut, lt.absmax, 64)
    assert np.array_equal(_bits(w), ref.view(np.uint16))


def test_dequant_fp16_rounding_cases():
    """Ties to even, +-inf on overflow, the smallest subnormal scale, q = z (W4); the
    LUT4 product rounded to fp32 and then to fp16 (a midpoint that ties to even)."""
    K, N = 256, 16
    codes = np.zeros((K, N), dtype=np.uint8)
    scales = np.full((2, N), np.float16(0.5), dtype=np.float16)
    zeros = np.zeros((2, N), dtype=np.float16)
    scales[:, 0] = np.array(0x2E66, dtype=np.uint16).view(np.float16)
    codes[:, 0] = 3
    scales[:, 1] = np.float16(65504)
    codes[:, 1] = 2
    scales[:, 9] = np.float16(65504)   # row gi + 8 of the fragment
    codes[:, 9] = 1
    zeros[:, 9] = 3
    scales[:, 3] = np.array(1, dtype=np.uint16).view(np.float16)
    codes[:, 3] = 5
    zeros[:, 3] = 8
    codes[:, 12] = 15
    zeros[:, 12] = 15
    codes[:, 14] = np.arange(K) % 16
    zeros[:, 14] = 7
    u = type("U", (), dict(bits=4, K=K, N=N, qweight=gen.pack_codes(codes, 4), scales=scales,
                           zeros=zeros))
    w = _bits(layers.from_uniform(u, DEV).dequant_fp16())
    with np.errstate(over="ignore"):
        ref = _oracle_w16(u).view(np.uint16)
    assert np.array_equal(w, ref)
    assert np.all(w[0] == 0x34CC) and np.all(w[1] == 0x7C00) and np.all(w[9] == 0xFC00)
    assert np.all(w[3] == 0x8003) and np.all(w[12] == 0x0000)

    # LUT4: lut = 1.5, absmax just above (2/3)(1 + 9 * 2^-11): the fp32 product is the fp16
    # midpoint 1 + 9 * 2^-11, which ties to 0x3C04
    a = np.float32(float(2 / 3 * (1 + 9 / 2048)))
    while float(a) * 1.5 <= 1 + 9 / 2048:
        a = np.nextafter(a, np.float32(2))
    lut = np.zeros(16, dtype=np.float16)
    lut[5] = np.float16(1.5)
    lcodes = np.full((K, N), 5, dtype=np.uint8)
    lt = type("L", (), dict(K=K, N=N, qbytes=gen.pack_nibbles(lcodes), lut=lut,
                            absmax=np.full((K // 64, N), a, dtype=np.float32)))
    wl = _bits(layers.from_lut4(lt, DEV).dequant_fp16())
    assert np.all(wl == 0x3C04)
    assert np.array_equal(wl, oracle.dequant_lut4_fp16_nk(lt.qbytes, lut, lt.absmax, 64)
                          .view(np.uint16))


def test_dequant_fp16_deterministic_and_overwrites():
    u = uniform_layer(777, 512, 208, 4)
    lay = layers.from_uniform(u, DEV)
    w = torch.full((208, 512), float("nan"), dtype=torch.float16, device=DEV)
    lay.dequant_fp16(w)
    first = _bits(w).copy()
    lay.dequant_fp16(w)
    assert np.array_equal(first, _bits(w))
    assert np.array_equal(first, _oracle_w16(u).view(np.uint16))


# ---------------------------------------------------------------------------
# prefill GEMM


@pytest.mark.parametrize("M", [1, 17, 64, 200])
@pytest.mark.parametrize("K,N", [(384, 208), (1024, 512), (2048, 1152)])
@pytest.mark.parametrize("fmt", ["w2", "w4", "w8", "lut4"])
def test_prefill_parity(fmt, K, N, M):
    if fmt == "lut4":
        lt = lut4_layer(611, K, N)
        lay = layers.from_lut4(lt, DEV)
        w16 = oracle.dequant_lut4_fp16_nk(lt.qbytes, lt.lut, lt.absmax, 64)
    else:
        bits = int(fmt[1:])
        u = uniform_layer(510 + bits, K, N, bits)
        lay = layers.from_uniform(u, DEV)
        w16 = _oracle_w16(u)
    x = gen.activations(900 + M, M, K)
    wbuf = torch.empty((N, K), dtype=torch.float16, device=DEV)
    y = lay.prefill(torch.from_numpy(x).to(DEV), w_fp16=wbuf)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(wbuf), w16.view(np.uint16))
    assert_parity(y.float().cpu().numpy(), oracle.prefill_matmul(x, w16), what=f"{fmt} M={M}")


# ---------------------------------------------------------------------------
# full size: the largest LLaMA-70B-shaped layer, sampled columns


@functools.lru_cache(maxsize=1)
def _big():
    K, N = 8192, 28672
    return gen.uniform_layer(gen.workload_seed(1, 4), K, N, 4)


@pytest.mark.slow
@pytest.mark.parametrize("M", [512])
def test_prefill_full_size_sampled(M):
    u = _big()
    K, N = u.K, u.N
    rs = np.random.default_rng(5)
    cols = np.unique(np.concatenate([rs.choice(N, 96, replace=False),
                                     [0, 15, 16, 127, 128, N - 129, N - 16, N - 1]]))
    lay = layers.from_uniform(u, DEV)
    x = gen.activations(4242, M, K)
    y = lay.prefill(torch.from_numpy(x).to(DEV))
    torch.cuda.synchronize()
    w_cols = lay._w_fp16[torch.from_numpy(cols).to(DEV)]
    ref16 = oracle.dequant_uniform_fp16_nk(u.qweight[:, cols], u.scales[:, cols],
                                           u.zeros[:, cols], 4, 128)
    assert np.array_equal(_bits(w_cols), ref16.view(np.uint16))
    assert_parity(y.float().cpu().numpy()[:, cols], oracle.prefill_matmul(x, ref16),
                  what=f"prefill {K}x{N} M={M}")
