"""The C-ABI library on a machine without a GPU: it loads, exports every declared
symbol, packs on the host, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ql():
    import weight_only_quantized_gemv_b200 as q
    return q


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)
    return [n for n in names if n not in ("if", "while")]


def test_exports_every_declared_symbol(ql):
    declared = _declared_functions()
    assert "qlinear_w4a16" in declared and "qlinear_pack" in declared
    lib = ctypes.CDLL(ql.LIBRARY_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(ql.EXPORTED)


def test_status_strings(ql):
    for s in range(8):
        assert ql._lib.ql_status_str(s)
    assert b"unknown" in ql._lib.ql_status_str(99)


@pytest.mark.parametrize("fmt,bits", [(2, 2), (4, 4), (8, 8), (16, 4)])
def test_pack_is_a_permutation_of_code_fields(ql, fmt, bits):
    K, N = 384, 208  # 13 tiles: one full 128-column block and a ragged one
    rs = np.random.default_rng(fmt)
    nbytes = K * N * bits // 8
    canon = rs.integers(0, 256, size=nbytes, dtype=np.uint8)
    packed = ql.qlinear_pack(fmt, canon, N, K)
    assert packed.nbytes == nbytes
    # multiset of code fields is preserved
    def fields(a):
        v = a.view(np.uint8)
        if bits == 8:
            return np.bincount(v, minlength=256)
        if bits == 4:
            return np.bincount(np.concatenate([v & 15, v >> 4]), minlength=16)
        return np.bincount(np.concatenate([(v >> s) & 3 for s in (0, 2, 4, 6)]), minlength=4)
    assert np.array_equal(fields(canon), fields(packed))
    # a single nonzero code lands in exactly one field
    one = np.zeros(nbytes, dtype=np.uint8)
    one[nbytes // 3] = 1
    p1 = ql.qlinear_pack(fmt, one, N, K)
    assert int(np.count_nonzero(p1)) == 1
    # deterministic
    assert np.array_equal(packed, ql.qlinear_pack(fmt, canon, N, K))


def test_pack_params_permutes(ql):
    K, N = 512, 48
    a = np.arange((K // 128) * N, dtype=np.float16).reshape(K // 128, N)
    p = ql.qlinear_pack_params(4, a, N, K)
    assert sorted(p.reshape(-1).tolist()) == sorted(a.reshape(-1).tolist())
    b = np.arange((K // 64) * N, dtype=np.float32).reshape(K // 64, N)
    q = ql.qlinear_pack_params(16, b, N, K)
    assert sorted(q.reshape(-1).tolist()) == sorted(b.reshape(-1).tolist())


def test_pack_tilecoo_reorders_tiles(ql):
    from synth import gen
    K, N = 384, 256
    lay = gen.outlier_layer(4100, K, N)
    o2, r2, v2 = ql.qlinear_pack_tilecoo(lay.tile_offsets, lay.tile_rc, lay.tile_vals, N, K)
    NB, KT = N // 128, K // 128
    for nt in range(NB):
        for kt in range(KT):
            t = kt * NB + nt
            t2 = nt * KT + kt
            a, b = lay.tile_offsets[t], lay.tile_offsets[t + 1]
            c, d = o2[t2], o2[t2 + 1]
            assert b - a == d - c
            assert np.array_equal(lay.tile_rc[a:b], r2[c:d])
            assert np.array_equal(lay.tile_vals[a:b].view(np.uint16), v2[c:d].view(np.uint16))
    bad = lay.tile_offsets.copy()
    bad[2], bad[3] = bad[3], bad[2] + 1
    with pytest.raises(ql.QLinearError):
        ql.qlinear_pack_tilecoo(bad, lay.tile_rc, lay.tile_vals, N, K)


def test_packer_rejects_bad_shapes(ql):
    assert ql.qlinear_packed_bytes(4, 24, 128) == 0
    assert ql.qlinear_packed_bytes(4, 16, 100) == 0
    assert ql.qlinear_packed_bytes(5, 16, 128) == 0
    assert ql.qlinear_packed_bytes(3, 16, 128) == 16 * 128 * 3 // 8
    assert ql.qlinear_packed_bytes(4, 16, 128) == 16 * 128 // 2
    assert ql._lib.qlinear_pack(4, None, None, 16, 128) == 1
    buf = np.zeros(64, dtype=np.uint8)
    assert ql._lib.qlinear_pack(4, buf.ctypes.data, buf.ctypes.data, 24, 128) == 2
    assert ql._lib.qlinear_pack(5, buf.ctypes.data, buf.ctypes.data, 16, 128) == 4


def test_hot_path_validates_before_any_device_work(ql):
    """Argument errors come back as status codes; no CUDA call is made for them."""
    lib = ql._lib
    a = 1 << 20  # an aligned, never-dereferenced address
    ok = dict(x=a, q=a, s=a, z=a, y=a, M=1, N=128, K=128, g=128, ws=a, wsb=1 << 20, st=None)

    def call(fn=lib.qlinear_w4a16, **kw):
        d = dict(ok, **kw)
        return fn(d["x"], d["q"], d["s"], d["z"], d["y"], d["M"], d["N"], d["K"], d["g"], d["ws"],
                  d["wsb"], d["st"])
    assert call(x=None) == 1
    assert call(y=None) == 1
    assert call(M=0) == 2 and call(M=17) == 2
    assert call(N=24) == 2 and call(K=100) == 2 and call(g=96) == 2 and call(g=256) == 2
    assert call(x=a + 2) == 3 and call(q=a + 16) == 3 and call(s=a + 2) == 3
    # scales and zeros are bulk-copied: 16-byte aligned sources only
    assert call(s=a + 4) == 3 and call(z=a + 8) == 3
    assert call(fn=lib.qlinear_w2a16, K=192) == 2
    assert call(fn=lib.qlinear_w8a16, N=8) == 2
    # LUT4 wants block 64
    assert lib.qlinear_lut4(a, a, a, a, a, 1, 128, 128, 128, a, 1 << 20, None) == 2
    # outliers need N % 128 == 0
    assert lib.qlinear_w4a16_outlier(a, a, a, a, a, a, a, a, 1, 144, 128, 128, a, 1 << 20, None) == 2
    assert lib.qlinear_w4a16_outlier(a, a, a, a, None, a, a, a, 1, 128, 128, 128, a, 1 << 20, None) == 1
    assert lib.qlinear_debug_unpack(4, None, a, 128, 128, None) == 1
    assert lib.qlinear_debug_unpack(5, a, a, 128, 128, None) == 4
    assert lib.qlinear_workspace_bytes(4, 0, 128, 128) == 0


def test_graft_entry_build_is_idempotent():
    import __graft_entry__ as ge
    ge.build()
    ge.build()


def test_prefill_entries_validate_before_any_device_work(ql):
    lib = ql._lib
    a = 1 << 20
    dq = lib.qlinear_dequant_fp16
    assert dq(3, a, a, a, a, 128, 128, None) == 4
    assert dq(4, None, a, a, a, 128, 128, None) == 1 and dq(4, a, a, a, None, 128, 128, None) == 1
    assert dq(4, a, a, a, a, 24, 128, None) == 2 and dq(4, a, a, a, a, 128, 100, None) == 2
    assert dq(4, a, a, a, a, 0, 128, None) == 2
    assert dq(4, a + 8, a, a, a, 128, 128, None) == 3 and dq(4, a, a, a, a + 8, 128, 128, None) == 3
    assert dq(4, a, a + 2, a, a, 128, 128, None) == 3 and dq(8, a, a, a + 2, a, 128, 128, None) == 3
    assert dq(16, a, a, a + 4, a, 128, 128, None) == 3 and dq(16, a, a + 1, a, a, 128, 128, None) == 3
    pf = lib.qlinear_prefill
    assert pf(5, a, a, a, a, a, a, 64, 128, 128, None) == 4
    assert pf(4, None, a, a, a, a, a, 64, 128, 128, None) == 1
    assert pf(4, a, a, a, a, a, None, 64, 128, 128, None) == 1
    assert pf(4, a, a, a, a, None, a, 64, 128, 128, None) == 1
    assert pf(4, a, a, a, a, a, a, 0, 128, 128, None) == 2
    assert pf(4, a, a, a, a, a, a, 64, 120, 128, None) == 2
    assert pf(4, a + 1, a, a, a, a, a, 64, 128, 128, None) == 3
    assert pf(4, a, a, a, a, a + 2, a, 64, 128, 128, None) == 3


def test_codebook_packers_and_checks(ql):
    K, N = 384, 96
    rs = np.random.default_rng(77)
    codes = rs.integers(0, 256, size=(K // 4, N), dtype=np.uint8)
    packed = ql.qlinear_pack_codebook(codes, N, K)
    assert packed.nbytes == codes.nbytes
    assert np.array_equal(np.sort(packed), np.sort(codes.reshape(-1)))
    # one marked code lands at the documented position: chunk (tile, group), lane, quad
    one = np.zeros_like(codes)
    j, n = 37, 70                   # group 1, slice 5; tile 2, lane 6
    one[j, n] = 1
    p1 = ql.qlinear_pack_codebook(one, N, K)
    G = K // 128
    ch = (n // 32) * G + j // 32
    jj, lane = j % 32, n % 32
    assert np.flatnonzero(p1).tolist() == [ch * 1024 + ((jj // 16) * 32 + lane) * 16 + jj % 16]
    s = np.arange((K // 128) * N, dtype=np.uint16).reshape(K // 128, N)
    ps = ql.qlinear_pack_codebook_scales(s, N, K)
    assert ps[((n // 32) * G + 2) * 32 + lane] == s[2, n]
    assert sorted(ps.tolist()) == sorted(s.reshape(-1).tolist())
    lib = ql._lib
    buf = np.zeros(64, dtype=np.uint8)
    assert lib.qlinear_pack_codebook(None, buf.ctypes.data, 32, 128) == 1
    assert lib.qlinear_pack_codebook(buf.ctypes.data, buf.ctypes.data, 48, 128) == 2
    a = 1 << 20
    cb = lib.qlinear_codebook
    assert cb(None, a, a, a, a, 1, 128, 128, a, 1 << 20, None) == 1
    assert cb(a, a, a, a, a, 5, 128, 128, a, 1 << 20, None) == 2
    assert cb(a, a, a, a, a, 0, 128, 128, a, 1 << 20, None) == 2
    assert cb(a, a, a, a, a, 1, 48, 128, a, 1 << 20, None) == 2
    assert cb(a, a, a, a, a, 1, 128, 100, a, 1 << 20, None) == 2
    assert cb(a, a + 8, a, a, a, 1, 128, 128, a, 1 << 20, None) == 3
    assert cb(a, a, a, a + 4, a, 1, 128, 128, a, 1 << 20, None) == 3
    assert cb(a + 1, a, a, a, a, 1, 128, 128, a, 1 << 20, None) == 3
    assert lib.qlinear_codebook_workspace_bytes(5, 128, 128) == 0


@pytest.mark.parametrize("fmt", [2, 4, 8])
def test_grouped_params_layout(ql, fmt):
    K, N = 384, 208          # 13 tiles: a full block and a ragged one; 3 units along K
    G = K // 128
    ntiles, nb = N // 16, (N // 16 + 7) // 8
    def chunk(b, g, jj):
        tb = min(8, ntiles - 8 * b)
        return b * G * 8 + g * tb + jj
    for group, ns in ((32, 4), (64, 2), (K, 1)):
        rows = 1 if group == K else K // group
        a = (np.arange(rows * N) % 2039).astype(np.float16).reshape(rows, N)
        p = ql.qlinear_pack_params_grouped(fmt, group, a, N, K)
        assert p.nbytes == ql.qlinear_params_bytes_grouped(fmt, group, N, K) == G * ns * N * 2
        for (b, g, jj, ss, gi, h) in [(0, 0, 0, 0, 0, 0), (1, 2, 4, ns - 1, 7, 1), (0, 1, 3, ns // 2, 5, 0)]:
            n = (8 * b + jj) * 16 + gi + 8 * h
            src = 0 if group == K else g * ns + ss
            assert p[(chunk(b, g, jj) * ns + ss) * 16 + gi * 2 + h] == a[src, n]
    # group 128 matches the ungrouped packer
    a = (np.arange(G * N) % 997).astype(np.float16).reshape(G, N)
    assert np.array_equal(ql.qlinear_pack_params_grouped(fmt, 128, a, N, K),
                          ql.qlinear_pack_params(fmt, a, N, K).reshape(-1))
    lib = ql._lib
    assert ql.qlinear_params_bytes_grouped(fmt, 96, N, K) == 0
    assert ql.qlinear_params_bytes_grouped(16, 64, N, K) == 0
    buf = np.zeros(64, dtype=np.uint16)
    assert lib.qlinear_pack_params_grouped(16, 64, buf.ctypes.data, buf.ctypes.data, N, K) == 4
    assert lib.qlinear_pack_params_grouped(fmt, 96, buf.ctypes.data, buf.ctypes.data, N, K) == 2
    assert lib.qlinear_pack_params_grouped(fmt, 64, None, buf.ctypes.data, N, K) == 1


def test_w3_packer_planes(ql):
    """The W3 packer puts each code's low two bits where W2 puts a code and its high bit in the
    second plane (word 4 + s / 4, bit 16 (dk & 1) + 4 (s % 4) + r8 / 8 + 2 (dk >> 1), after
    the 512 bytes of quads): decoding that layout gives back the canonical codes."""
    import oracle
    from synth import gen
    K, N = 384, 208
    rs = np.random.default_rng(3)
    codes = rs.integers(0, 8, size=(K, N), dtype=np.uint8)
    canon = gen.pack_codes(codes, 3)
    assert ql.qlinear_packed_bytes(3, N, K) == canon.nbytes == K * N * 3 // 8
    packed = ql.qlinear_pack(3, canon, N, K).view(np.uint32)
    assert np.array_equal(oracle.unpack_uniform(canon, 3), codes)
    G, ntiles = K // 128, N // 16
    out = np.zeros_like(codes)
    for b in range((ntiles + 7) // 8):
        tb = min(8, ntiles - 8 * b)
        for g in range(G):
            for jj in range(tb):
                ch = packed[(b * G * 8 + g * tb + jj) * 192:][:192]
                for lane in range(32):
                    gi, t = lane >> 2, lane & 3
                    w = [int(ch[lane * 4 + i]) for i in range(4)] + \
                        [int(ch[128 + 2 * lane + i]) for i in range(2)]
                    for s in range(8):
                        for dk in range(4):
                            for hi in (0, 1):
                                k = g * 128 + 32 * (s >> 1) + 8 * t + 4 * (s & 1) + dk
                                n = (8 * b + jj) * 16 + gi + 8 * hi
                                # W2 position of the low bits (layout.h)
                                q2 = (w[s >> 1] >> (16 * (dk & 1) + 8 * (dk >> 1) + 2 * hi + 4 * (s & 1))) & 3
                                q1 = (w[4 + (s >> 2)] >> (16 * (dk & 1) + 4 * (s & 3) + hi + 2 * (dk >> 1))) & 1
                                out[k, n] = q2 + 4 * q1
    assert np.array_equal(out, codes)
    lib = ql._lib
    a = 1 << 20
    assert lib.qlinear_w3a16(a, a, a, a, a, 1, 128, 128, 64, a, 1 << 20, None) == 2   # group 64
    assert lib.qlinear_w3a16(None, a, a, a, a, 1, 128, 128, 128, a, 1 << 20, None) == 1
    assert ql.qlinear_params_bytes_grouped(3, 64, N, K) == 0
    assert ql.qlinear_params_bytes_grouped(3, K, N, K) == G * N * 2


def test_pack_codebook_tc_layout(ql):
    """Byte 2 s + r of lane l in chunk (block b, group g, tile jj) is the code of the 4-vector
    that holds k = 128 g + 32 (s // 2) + 8 (l % 4) + 4 (s % 2) of column
    16 (8 b + jj) + l // 4 + 8 r (the fragment k order of the GEMV)."""
    K, N = 256, 160  # 2 groups, 10 tiles: a full block and a ragged one of 2 tiles
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, size=(K // 4, N), dtype=np.uint8)
    packed = ql.qlinear_pack_codebook_tc(codes, N, K)
    G, ntiles = K // 128, N // 16
    seen = 0
    for b in range(2):
        tb = min(8, ntiles - 8 * b)
        for g in range(G):
            for jj in range(tb):
                c = b * G * 8 + g * tb + jj
                for lane in (0, 5, 18, 31):
                    for s in range(8):
                        for r in range(2):
                            k = 128 * g + 32 * (s // 2) + 8 * (lane % 4) + 4 * (s % 2)
                            n = 16 * (8 * b + jj) + lane // 4 + 8 * r
                            assert packed[c * 512 + lane * 16 + 2 * s + r] == codes[k // 4, n]
                            seen += 1
    assert seen == (8 + 2) * G * 4 * 16
    assert sorted(packed.tolist()) == sorted(codes.ravel().tolist())  # a permutation
