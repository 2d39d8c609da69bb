"""CUDA path against the fp64 oracle, element by element, through the C ABI.

* decode: packed codes and dequantized weights, bit-exact;
* GEMV: every format and M bucket, shapes spanning several tiles and blocks with
  ragged tails, many split-K partitions;
* special cases: x = 0, one-hot x (bit-exact), codes at the zero point, outlier-only;
* determinism and workspace reuse.
"""
import os

import numpy as np
import pytest

import oracle
from synth import gen
from tests.helpers import assert_parity, lut4_layer, outlier_layer, uniform_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from weight_only_quantized_gemv_b200 import layers
    import weight_only_quantized_gemv_b200 as ql

DEV = "cuda:0"
FORMATS = [("w2", 2), ("w4", 4), ("w8", 8)]
SHAPES = [(128, 16), (640, 208), (1024, 512), (2048, 1152)]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def _x(seed, M, K):
    x = gen.activations(seed, M, K)
    return x, torch.from_numpy(x).to(DEV)


def _np(t):
    torch.cuda.synchronize()
    return t.float().cpu().numpy()


def _fwd(lay, xd):
    """lay.forward, then the check that every device wait of the call completed."""
    y = _np(lay.forward(xd))
    assert lay.read_error() == 0, "a device wait gave up"
    return y


# ---------------------------------------------------------------------------
# decode, bit-exact


@pytest.mark.parametrize("K,N", [(256, 48), (640, 208), (1024, 512)])
@pytest.mark.parametrize("name,bits", FORMATS)
def test_debug_unpack_and_dequant_bit_exact(name, bits, K, N):
    u = uniform_layer(100 + bits, K, N, bits)
    lay = layers.from_uniform(u, DEV)
    codes = lay.debug_unpack().cpu().numpy()
    assert np.array_equal(codes, oracle.unpack_uniform(u.qweight, bits))
    w = lay.debug_dequant().cpu().numpy()
    ref = oracle.dequant_uniform(oracle.unpack_uniform(u.qweight, bits), u.scales, u.zeros, 128)
    assert np.array_equal(w, ref.astype(np.float32))
    assert np.array_equal(ref.astype(np.float32).astype(np.float64), ref)  # exact in fp32


@pytest.mark.parametrize("K,N", [(256, 48), (640, 208)])
def test_debug_lut4_bit_exact(K, N):
    lt = lut4_layer(301, K, N)
    lay = layers.from_lut4(lt, DEV)
    codes = lay.debug_unpack().cpu().numpy()
    assert np.array_equal(codes, oracle.unpack_lut4(lt.qbytes))
    w = lay.debug_dequant().cpu().numpy()
    ref = oracle.dequant_lut4_fp32(oracle.unpack_lut4(lt.qbytes), lt.lut, lt.absmax, 64)
    assert np.array_equal(w, ref)


# ---------------------------------------------------------------------------
# GEMV parity


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("name,bits", FORMATS)
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 13, 16])
def test_uniform_gemv_parity(name, bits, K, N, M):
    u = uniform_layer(200 + bits, K, N, bits)
    lay = layers.from_uniform(u, DEV)
    x, xd = _x(200 + M, M, K)
    y = _fwd(lay, xd)
    assert_parity(y, oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, bits, 128),
                  what=f"{name} M={M} K={K} N={N}")


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("M", [1, 4, 8, 9, 16])
def test_lut4_gemv_parity(K, N, M):
    lt = lut4_layer(400, K, N)
    lay = layers.from_lut4(lt, DEV)
    x, xd = _x(400 + M, M, K)
    y = _fwd(lay, xd)
    assert_parity(y, oracle.gemv_lut4(x, lt.qbytes, lt.lut, lt.absmax, 64), what=f"lut4 M={M}")


@pytest.mark.parametrize("K,N", [(512, 384), (1024, 1024), (2048, 256)])
@pytest.mark.parametrize("M", [1, 2, 4, 8, 16])
def test_outlier_gemv_parity(K, N, M):
    o = outlier_layer(500, K, N)
    lay = layers.from_outlier(o, DEV)
    x, xd = _x(500 + M, M, K)
    y = _fwd(lay, xd)
    ref = oracle.gemv_outlier(x, o.dense.qweight, o.dense.scales, o.dense.zeros, o.tile_offsets,
                              o.tile_rc, o.tile_vals, 4, 128)
    assert_parity(y, ref, what=f"outlier M={M} K={K} N={N}")


@pytest.mark.parametrize("cap", ["1", "2", "3", "5", "7", "13", "29", "64"])
@pytest.mark.parametrize("kind", ["w4", "w2", "lut4", "outlier"])
def test_split_k_partitions(kind, cap):
    """The persistent grid capped at a few CTAs: ranges that cut blocks in many places."""
    K, N, M = 1408, 416, 3  # 11 groups, 26 tiles = 3 full blocks + a ragged one
    if kind == "outlier":
        K, N = 1408, 384
    old = os.environ.get("QLINEAR_MAX_CTAS")
    os.environ["QLINEAR_MAX_CTAS"] = cap
    try:
        x, xd = _x(600, M, K)
        if kind == "lut4":
            lt = lut4_layer(601, K, N)
            lay = layers.from_lut4(lt, DEV)
            ref = oracle.gemv_lut4(x, lt.qbytes, lt.lut, lt.absmax, 64)
        elif kind == "outlier":
            o = outlier_layer(602, K, N)
            lay = layers.from_outlier(o, DEV)
            ref = oracle.gemv_outlier(x, o.dense.qweight, o.dense.scales, o.dense.zeros,
                                      o.tile_offsets, o.tile_rc, o.tile_vals, 4, 128)
        else:
            bits = 4 if kind == "w4" else 2
            u = uniform_layer(603, K, N, bits)
            lay = layers.from_uniform(u, DEV)
            ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, bits, 128)
        assert ql.qlinear_plan(4, M, N, K).ctas == min(int(cap), (N // 128 + 1) * (K // 128)) \
            or kind != "w4"
        for _ in range(2):  # the second call checks that the counters were reset
            y = _fwd(lay, xd)
            assert_parity(y, ref, what=f"{kind} cap={cap}")
    finally:
        if old is None:
            os.environ.pop("QLINEAR_MAX_CTAS", None)
        else:
            os.environ["QLINEAR_MAX_CTAS"] = old


@pytest.mark.parametrize("wpu", ["1", "2", "4"])
@pytest.mark.parametrize("cap", ["0", "7", "29"])
@pytest.mark.parametrize("M", [1, 5, 8])
def test_w4_warps_per_unit(wpu, cap, M):
    """Every W4 M <= 8 variant (1, 2 or 4 warps per unit), whole-block and split-K grids,
    on a ragged block."""
    K, N = 1408, 416
    env = {"QLINEAR_WPU": wpu, "QLINEAR_MAX_CTAS": cap}
    old = {k: os.environ.get(k) for k in env}
    os.environ.update(env)
    try:
        u = uniform_layer(610, K, N, 4)
        lay = layers.from_uniform(u, DEV)
        x, xd = _x(611 + M, M, K)
        ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 4, 128)
        assert ql.qlinear_plan(4, M, N, K).warps_per_unit == int(wpu)
        for _ in range(2):
            assert_parity(_fwd(lay, xd), ref, what=f"w4 wpu={wpu} cap={cap} M={M}")
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


# ---------------------------------------------------------------------------
# special cases


@pytest.mark.parametrize("name,bits", FORMATS)
def test_zero_x_gives_zero(name, bits):
    K, N = 640, 208
    lay = layers.from_uniform(uniform_layer(700, K, N, bits), DEV)
    y = lay.forward(torch.zeros((4, K), dtype=torch.float16, device=DEV))
    assert torch.count_nonzero(y).item() == 0


@pytest.mark.parametrize("name,bits", FORMATS)
def test_one_hot_x_is_bit_exact(name, bits):
    """x = e_k: y[m, n] = fp16(s (q[k, n] - z)); one exact fp32 product, one rounding."""
    K, N = 640, 208
    u = uniform_layer(710, K, N, bits)
    lay = layers.from_uniform(u, DEV)
    ks = [0, 1, 2, 3, 7, 100, 129, 255, 383, 639]
    x = np.zeros((len(ks) if len(ks) <= 16 else 16, K), dtype=np.float16)
    for m, k in enumerate(ks):
        x[m, k] = 1
    y = lay.forward(torch.from_numpy(x).to(DEV)).cpu().numpy()
    deq = oracle.dequant_uniform(oracle.unpack_uniform(u.qweight, bits), u.scales, u.zeros, 128)
    for m, k in enumerate(ks):
        assert np.array_equal(y[m].view(np.uint16), deq[k].astype(np.float16).view(np.uint16)), (m, k)


def test_one_hot_lut4():
    K, N = 640, 208
    lt = lut4_layer(720, K, N)
    lay = layers.from_lut4(lt, DEV)
    ks = [0, 1, 5, 63, 64, 200, 639]
    x = np.zeros((len(ks), K), dtype=np.float16)
    for m, k in enumerate(ks):
        x[m, k] = 1
    y = lay.forward(torch.from_numpy(x).to(DEV)).cpu().numpy()
    deq32 = oracle.dequant_lut4_fp32(oracle.unpack_lut4(lt.qbytes), lt.lut, lt.absmax, 64)
    for m, k in enumerate(ks):
        assert np.array_equal(y[m].view(np.uint16), deq32[k].astype(np.float16).view(np.uint16))


def test_codes_at_zero_point_cancel_and_outlier_only_is_exact():
    K, N = 512, 256
    o = outlier_layer(730, K, N)
    d = o.dense
    zcodes = np.repeat(d.zeros.astype(np.uint8), 128, axis=0)
    qz = gen.pack_codes(zcodes, 4)
    dense = ql.layers.QuantLinear(4, K, N, qz, d.scales, d.zeros, device=DEV)
    x, xd = _x(731, 5, K)
    # The deferred form computes sum_k z x - z sum_k x: it cancels up to fp32 rounding of the
    # two sums (eager dequantization would give exact zeros).  Bound: a few fp32 ulps of
    # s * z * sum_k |x| per group.
    y = _fwd(dense, xd)
    s = d.scales.astype(np.float64)
    z = d.zeros.astype(np.float64)
    xa = np.abs(x.astype(np.float64)).reshape(5, K // 128, 128).sum(axis=2)
    bound = (xa @ (s * z)) * 2.0 ** -20 + 2.0 ** -24
    assert np.all(np.abs(y) <= bound), float(np.max(np.abs(y) / bound))
    # outlier-only: one-hot x picks single fp16 outlier values exactly
    lay = ql.layers.QuantLinear(4, K, N, qz, d.scales, d.zeros,
                                tilecoo=(o.tile_offsets, o.tile_rc, o.tile_vals), device=DEV)
    dense_o = oracle.tilecoo_to_dense(o.tile_offsets, o.tile_rc, o.tile_vals, K, N)
    ks = sorted(set((o.positions // N)[:6].tolist()))
    x1 = np.zeros((len(ks), K), dtype=np.float16)
    for m, k in enumerate(ks):
        x1[m, k] = 1
    y = lay.forward(torch.from_numpy(x1).to(DEV)).cpu().numpy()
    for m, k in enumerate(ks):
        assert np.array_equal(y[m].view(np.uint16), dense_o[k].astype(np.float16).view(np.uint16))


def test_linearity_in_x():
    K, N = 1024, 512
    lay = layers.from_uniform(uniform_layer(740, K, N, 4), DEV)
    xa, xad = _x(741, 2, K)
    xb, xbd = _x(742, 2, K)
    ya = _np(lay.forward(xad))
    yb = _np(lay.forward(xbd))
    yab = _np(lay.forward(torch.cat([xad, xbd])))
    assert np.array_equal(yab, np.concatenate([ya, yb]))  # rows are independent


def test_deterministic_and_workspace_reuse():
    K, N = 2048, 1152
    a = layers.from_uniform(uniform_layer(750, K, N, 4), DEV)
    b = layers.from_uniform(uniform_layer(751, 1024, 512, 2), DEV)
    b.workspace = a.workspace  # one workspace shared by two layers on one stream
    _, xd = _x(752, 3, K)
    _, xb = _x(753, 3, 1024)
    y1 = a.forward(xd).clone()
    b.forward(xb)
    y2 = a.forward(xd).clone()
    assert torch.equal(y1, y2)
    torch.cuda.synchronize()


def test_explicit_stream():
    K, N = 1024, 512
    u = uniform_layer(760, K, N, 4)
    lay = layers.from_uniform(u, DEV)
    x, xd = _x(761, 1, K)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = lay.forward(xd, stream=s)
    s.synchronize()
    assert_parity(y.float().cpu().numpy(), oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 4, 128))


def test_workspace_too_small_is_rejected():
    K, N = 1024, 512
    lay = layers.from_uniform(uniform_layer(770, K, N, 4), DEV)
    lay.workspace = lay.workspace[:4]
    with pytest.raises(ql.QLinearError) as e:
        lay.forward(torch.zeros((1, K), dtype=torch.float16, device=DEV))
    assert e.value.status == 5


@pytest.mark.parametrize("kind,M", [("w4", 1), ("w2", 1), ("w4", 16), ("lut4", 1), ("outlier", 8)])
def test_many_launches_bit_identical(kind, M):
    """A stage refilled before every lane has read it would show as results that differ
    between launches: 200 back-to-back launches on a layer whose CTAs each stream many units
    (every ring wraps), all bit-identical to the first, the first within tolerance.  The
    outlier kernel adds its outliers with shared-memory float atomics, whose order varies
    between launches: there each launch must stay within tolerance and within one fp16
    rounding of the first."""
    K, N = 4096, 2048
    x, xd = _x(773 + M, M, K)
    if kind == "lut4":
        L = lut4_layer(770, K, N)
        lay = layers.from_lut4(L, DEV)
        want = oracle.gemv_lut4(x, L.qbytes, L.lut, L.absmax, 64)
    elif kind == "outlier":
        o = outlier_layer(771, K, N)
        lay = layers.from_outlier(o, DEV)
        want = oracle.gemv_outlier(x, o.dense.qweight, o.dense.scales, o.dense.zeros,
                                   o.tile_offsets, o.tile_rc, o.tile_vals, 4, 128)
    else:
        bits = int(kind[1:])
        u = uniform_layer(772, K, N, bits)
        lay = layers.from_uniform(u, DEV)
        want = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, bits, 128)
    y = torch.empty((M, N), dtype=torch.float16, device=DEV)
    lay.forward(xd, y)
    torch.cuda.synchronize()
    first = y.view(torch.int16).cpu().numpy().copy()
    assert_parity(first.view(np.float16).astype(np.float64), want, what=f"{kind} M={M}")
    f0 = first.view(np.float16).astype(np.float64)
    for _ in range(200):
        lay.forward(xd, y)
        torch.cuda.synchronize()
        h = y.view(torch.int16).cpu().numpy()
        if kind != "outlier":
            assert np.array_equal(h, first)
        else:
            f = h.view(np.float16).astype(np.float64)
            assert np.all(np.abs(f - f0) <= 2.0 ** -10 * np.abs(f0) + 2.0 ** -24)
            assert_parity(f, want, what=f"{kind} M={M}, repeated")
    assert lay.read_error() == 0
