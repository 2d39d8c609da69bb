"""Seeded generators for the five quantized-GEMV workloads.

Every array is drawn from ``numpy.random.default_rng([seed, stream])`` with a
fixed stream per quantity, so any consumer can regenerate the same input from
``(seed, shape)`` alone.  ``seed = 1000 * workload + layer``.

What is produced, and the recipe each follows
---------------------------------------------
* fp32 weights ``W[K, N] ~ N(0, 0.02)`` (0.02 is the standard deviation).
* fp16 activations ``x[M, K] ~ N(0, 1)``, rounded to nearest-even.
* Group-wise asymmetric min-max codes for b = 2, 4, 8 bits with a group of
  128 along K per output column (QFactory page, "问题与动机" and observation 1:
  GPTQ-style fine-grained asymmetric group quantization, group size 128).
  Per (group, column): ``s32 = fp32(max - min) / fp32(2^b - 1)``, the stored
  scale is ``s = fp16(s32)``, ``z = clip(rint(-min / s), 0, 2^b - 1)`` and
  ``q = clip(rint(w / s) + z, 0, 2^b - 1)``, the last two in fp64 with the
  stored fp16 ``s``.  A group whose stored scale is 0 stores s = z = q = 0.
* Canonical code layout ``uint32[K * b / 32, N]``: each column's codes form one
  little-endian bit stream along K, code k in bits ``[b*k, b*k + b)``, 32 bits per
  word.  For b = 2, 4, 8 word ``(j, n)`` bits ``[b*i, b*i + b)`` hold
  ``q[P*j + i, n]`` (``P = 32 / b``); 3-bit codes (b = 3, the GPTQ-style packing
  of 32 codes in 3 words) run across word boundaries.
* LUT4 (the NF4-style format of the "Fast NF4 Dequantization Kernels" page):
  a sorted 16-entry fp16 table holding -1, 0, +1 and 13 further distinct
  values drawn from U(-1, 1); an fp32 ``absmax`` per 64-element block along K
  per column; each code is the index of the table entry nearest to
  ``w / absmax`` (fp64, lower index on a tie, the index of 0.0 when
  absmax = 0); two codes per byte, low nibble = even k.
* Outlier-aware W4 (the FlashQuant page, English abstract): 0.5% of the
  weights, drawn uniformly without replacement, are scaled by 10 and kept as
  fp16 in Tile-COO with 128 x 128 (K x N) tiles; the remaining weights are
  min-max quantized over the non-outlier entries of each group, and each
  outlier's dense slot holds the group's zero code.

* Codebook (the CodeGEMM page's m1v4g128 configuration: one codebook, vectors
  of 4 weights along K, 8-bit codes, group normalization over 128 weights): a
  256 x 4 fp16 codebook with entries from U(-1, 1).  The page's codebooks come
  from K-means/AQLM calibration, which is training and out of scope; the
  GEMV's arithmetic does not depend on how the codes were chosen.  By default
  the codes are uniform random bytes and each (group, column) scale is
  ``fp16(0.02 * (2.5 + U(0, 1)))`` (about the absmax of 128 N(0, 0.02)
  draws); given weights ``w`` (small sizes), the scale is the group's fp16
  absmax and each code is the centroid nearest to the normalized 4-vector
  ``w / s`` (squared distance in fp64, lower index on a tie).

None of these functions unpack codes, dequantize or multiply by x.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

STREAM_W = 0
STREAM_X = 1
STREAM_OUTLIER = 2
STREAM_LUT = 3
STREAM_CB = 4

GROUP = 128
LUT_BLOCK = 64
TILE = 128
OUTLIER_FRACTION = 0.005
OUTLIER_SCALE = 10.0
CB_VEC = 4          # weights per codebook vector (along K)
CB_ENTRIES = 256    # 8-bit codes


def workload_seed(workload: int, layer: int) -> int:
    return 1000 * workload + layer


def rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, stream])


def weights(seed: int, K: int, N: int) -> np.ndarray:
    """fp32 ``W[K, N]`` with entries N(0, 0.02)."""
    return rng(seed, STREAM_W).standard_normal((K, N), dtype=np.float32) * np.float32(0.02)


def activations(seed: int, M: int, K: int) -> np.ndarray:
    """fp16 ``x[M, K]``: fp32 N(0, 1) draws rounded to fp16 (nearest-even)."""
    return rng(seed, STREAM_X).standard_normal((M, K), dtype=np.float32).astype(np.float16)


# ---------------------------------------------------------------------------
# canonical code packing (little-endian fields along K)


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """``uint8[K, N]`` codes -> canonical ``uint32[K * bits / 32, N]``: each column is one
    little-endian bit stream, code k in bits ``[bits*k, bits*k + bits)``, 32 bits per word.
    For bits dividing 32 that is ``P = 32 / bits`` whole codes per word; 3-bit codes run
    across word boundaries (32 codes in 3 words)."""
    K, N = codes.shape
    if (K * bits) % 32:
        raise ValueError("K * bits must be a multiple of 32")
    if 32 % bits == 0:
        P = 32 // bits
        c = codes.reshape(K // P, P, N).astype(np.uint32)
        out = np.zeros((K // P, N), dtype=np.uint32)
        for i in range(P):
            out |= c[:, i, :] << np.uint32(bits * i)
        return out
    W = K * bits // 32
    out = np.zeros((W + 1, N), dtype=np.uint64)     # one spare word for the last straddle
    c = codes.astype(np.uint64)
    for k in range(K):
        o = bits * k
        j, sh = o // 32, o % 32
        out[j] |= (c[k] << np.uint64(sh)) & np.uint64(0xFFFFFFFF)
        if sh + bits > 32:
            out[j + 1] |= c[k] >> np.uint64(32 - sh)
    return out[:W].astype(np.uint32)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """``uint8[K, N]`` 4-bit codes -> canonical LUT4 bytes ``uint8[K / 2, N]``
    (low nibble = even k, high nibble = odd k)."""
    K, N = codes.shape
    c = codes.reshape(K // 2, 2, N)
    return (c[:, 0, :] | (c[:, 1, :] << 4)).astype(np.uint8)


# ---------------------------------------------------------------------------
# group-wise asymmetric min-max quantization (input recipe of the workloads)


@dataclasses.dataclass
class UniformLayer:
    bits: int
    K: int
    N: int
    group: int
    codes: np.ndarray      # uint8[K, N] (kept for the generator's own checks)
    qweight: np.ndarray    # uint32[K * bits / 32, N] canonical
    scales: np.ndarray     # fp16[K / group, N]
    zeros: np.ndarray      # fp16[K / group, N] (integers)
    scales32: np.ndarray   # fp32[K / group, N]: the pre-rounding fp32 scale


def _quantize_minmax(w: np.ndarray, bits: int, group: int,
                     mask: Optional[np.ndarray] = None):
    """Codes, fp16 scales, fp16 zeros and fp32 pre-rounding scales.

    ``mask`` (same shape as ``w``, True = excluded) removes entries from the
    min/max of their group; excluded entries get the group's zero code.
    """
    K, N = w.shape
    G = K // group
    qmax = (1 << bits) - 1
    wg = w.reshape(G, group, N)
    if mask is None:
        mn = wg.min(axis=1)
        mx = wg.max(axis=1)
    else:
        mg = mask.reshape(G, group, N)
        mn = np.where(mg, np.float32(np.inf), wg).min(axis=1)
        mx = np.where(mg, np.float32(-np.inf), wg).max(axis=1)
        allout = ~np.isfinite(mn)
        mn = np.where(allout, np.float32(0), mn).astype(np.float32)
        mx = np.where(allout, np.float32(0), mx).astype(np.float32)
    s32 = (mx - mn).astype(np.float32) / np.float32(qmax)
    s16 = s32.astype(np.float16)
    s64 = s16.astype(np.float64)
    ok = s64 > 0
    safe = np.where(ok, s64, 1.0)
    z = np.where(ok, np.clip(np.rint(-mn.astype(np.float64) / safe), 0, qmax), 0.0)
    codes = np.empty((G, group, N), dtype=np.uint8)
    for g in range(G):  # one group row at a time keeps fp64 temporaries small
        q = np.rint(wg[g].astype(np.float64) / safe[g]) + z[g]
        q = np.clip(q, 0, qmax)
        q = np.where(ok[g], q, 0.0)
        if mask is not None:
            q = np.where(mg[g], z[g], q)
        codes[g] = q.astype(np.uint8)
    return codes.reshape(K, N), s16, z.astype(np.float16), s32


def uniform_layer(seed: int, K: int, N: int, bits: int, group: int = GROUP,
                  w: Optional[np.ndarray] = None) -> UniformLayer:
    if w is None:
        w = weights(seed, K, N)
    codes, s16, z16, s32 = _quantize_minmax(w, bits, group)
    return UniformLayer(bits, K, N, group, codes, pack_codes(codes, bits), s16, z16, s32)


# ---------------------------------------------------------------------------
# LUT4 (NF4-style) quantization


@dataclasses.dataclass
class Lut4Layer:
    K: int
    N: int
    block: int
    codes: np.ndarray     # uint8[K, N]
    qbytes: np.ndarray    # uint8[K / 2, N] canonical
    lut: np.ndarray       # fp16[16], sorted ascending
    absmax: np.ndarray    # fp32[K / block, N]


def lut16(seed: int) -> np.ndarray:
    """Sorted fp16 table: -1, 0, +1 and 13 distinct fp16 draws from U(-1, 1)."""
    r = rng(seed, STREAM_LUT)
    vals = {np.float16(-1.0), np.float16(0.0), np.float16(1.0)}
    while len(vals) < 16:
        v = np.float16(r.uniform(-1.0, 1.0))
        if v == 0:  # -0.0 and 0.0 compare equal: keep a single zero entry
            continue
        vals.add(v)
    return np.array(sorted(vals, key=float), dtype=np.float16)


def _nearest_lut_codes(r: np.ndarray, lut: np.ndarray) -> np.ndarray:
    """Index of the nearest table entry for each ratio (fp64 distances), lower index on ties.

    The table is sorted, so |r - lut[c]| (fp64) does not increase towards r from either
    side: the minimum is one of the two entries around r's insertion point.
    """
    lut64 = lut.astype(np.float64)
    hi = np.clip(np.searchsorted(lut64, r, side="left"), 1, 15)
    lo = hi - 1
    dlo = np.abs(r - lut64[lo])
    dhi = np.abs(r - lut64[hi])
    return np.where(dlo <= dhi, lo, hi).astype(np.uint8)


def lut4_layer(seed: int, K: int, N: int, block: int = LUT_BLOCK,
               w: Optional[np.ndarray] = None, lut: Optional[np.ndarray] = None) -> Lut4Layer:
    if w is None:
        w = weights(seed, K, N)
    if lut is None:
        lut = lut16(seed)
    B = K // block
    wb = w.reshape(B, block, N)
    absmax = np.abs(wb).max(axis=1).astype(np.float32)
    zero_idx = int(np.nonzero(lut.astype(np.float64) == 0.0)[0][0])
    codes = np.empty((B, block, N), dtype=np.uint8)
    for b in range(B):
        a = absmax[b].astype(np.float64)
        ok = a > 0
        r = wb[b].astype(np.float64) / np.where(ok, a, 1.0)
        c = _nearest_lut_codes(r, lut)
        codes[b] = np.where(ok, c, np.uint8(zero_idx))
    codes = codes.reshape(K, N)
    return Lut4Layer(K, N, block, codes, pack_nibbles(codes), lut, absmax)


# ---------------------------------------------------------------------------
# outlier-aware W4 with Tile-COO


@dataclasses.dataclass
class OutlierLayer:
    dense: UniformLayer
    positions: np.ndarray     # int64[nnz] flat indices k * N + n, ascending
    tile_offsets: np.ndarray  # uint32[T + 1]
    tile_rc: np.ndarray       # uint8[nnz, 2] (row, col) inside the tile
    tile_vals: np.ndarray     # fp16[nnz]
    w_full: np.ndarray        # fp32[K, N] weights after the x10 outlier scaling


def outlier_count(K: int, N: int) -> int:
    return int(round(OUTLIER_FRACTION * K * N))


def outlier_layer(seed: int, K: int, N: int, bits: int = 4, group: int = GROUP,
                  w: Optional[np.ndarray] = None, nnz: Optional[int] = None) -> OutlierLayer:
    if K % TILE or N % TILE:
        raise ValueError("outlier layers need K and N to be multiples of 128")
    if w is None:
        w = weights(seed, K, N)
    if nnz is None:
        nnz = outlier_count(K, N)
    pos = np.sort(rng(seed, STREAM_OUTLIER).choice(K * N, size=nnz, replace=False)).astype(np.int64)
    w_full = w.copy()
    flat = w_full.reshape(-1)
    flat[pos] = flat[pos] * np.float32(OUTLIER_SCALE)
    mask = np.zeros(K * N, dtype=bool)
    mask[pos] = True
    mask = mask.reshape(K, N)
    codes, s16, z16, s32 = _quantize_minmax(w_full, bits, group, mask=mask)
    dense = UniformLayer(bits, K, N, group, codes, pack_codes(codes, bits), s16, z16, s32)
    k = pos // N
    n = pos % N
    kt, nt = k // TILE, n // TILE
    tiles_n = N // TILE
    t = kt * tiles_n + nt
    order = np.lexsort((n % TILE, k % TILE, t))  # by tile, then row, then col
    t, k, n = t[order], k[order], n[order]
    T = (K // TILE) * tiles_n
    counts = np.bincount(t, minlength=T)
    offsets = np.zeros(T + 1, dtype=np.uint32)
    offsets[1:] = np.cumsum(counts).astype(np.uint32)
    rc = np.stack([k % TILE, n % TILE], axis=1).astype(np.uint8)
    vals = w_full[k, n].astype(np.float16)
    return OutlierLayer(dense, pos, offsets, rc, vals, w_full)


# ---------------------------------------------------------------------------
# the five workloads (shapes as (K, N))

LLAMA_SHAPES = [(4096, 12288), (4096, 4096), (4096, 28672), (14336, 4096),
                (8192, 28672), (28672, 8192)]

WORKLOADS = {
    0: dict(kind="w4", shapes=[(4096, 4096)], M=[1]),
    1: dict(kind="w4", shapes=LLAMA_SHAPES, M=[1]),
    2: dict(kind="w2", shapes=LLAMA_SHAPES, M=[1], w8_shapes=[(4096, 28672), (8192, 28672)]),
    3: dict(kind="lut4", shapes=[(8192, 28672), (28672, 8192)], M=[1]),
    4: dict(kind="outlier", shapes=[(4096, 14336), (8192, 28672)], M=[1, 2, 4, 8, 16]),
}


# ---------------------------------------------------------------------------
# codebook (vector) quantization, m = 1 codebook, v = 4, b = 8


@dataclasses.dataclass
class CodebookLayer:
    K: int
    N: int
    group: int
    codebook: np.ndarray   # fp16[256, 4]
    codes: np.ndarray      # uint8[K / 4, N]: code of the 4-vector (4j .. 4j + 3, n)
    scales: np.ndarray     # fp16[K / group, N]


def codebook_layer(seed: int, K: int, N: int, group: int = GROUP,
                   w: Optional[np.ndarray] = None) -> CodebookLayer:
    r = rng(seed, STREAM_CB)
    codebook = r.uniform(-1.0, 1.0, size=(CB_ENTRIES, CB_VEC)).astype(np.float16)
    if w is None:
        codes = r.integers(0, CB_ENTRIES, size=(K // CB_VEC, N), dtype=np.uint8)
        scales = (0.02 * (2.5 + r.uniform(0.0, 1.0, size=(K // group, N)))).astype(np.float16)
        return CodebookLayer(K, N, group, codebook, codes, scales)
    G = K // group
    wg = w.astype(np.float64).reshape(G, group, N)
    scales = np.abs(wg).max(axis=1).astype(np.float16)
    s = scales.astype(np.float64)
    ok = s > 0
    u = wg / np.where(ok, s, 1.0)[:, None, :]                      # [G, group, N]
    vec = u.reshape(G, group // CB_VEC, CB_VEC, N).transpose(0, 1, 3, 2).reshape(-1, CB_VEC)
    c = codebook.astype(np.float64)
    d = ((vec[:, None, :] - c[None, :, :]) ** 2).sum(axis=2)        # [vectors, 256]
    idx = d.argmin(axis=1).astype(np.uint8)                         # first minimum on a tie
    codes = idx.reshape(G, group // CB_VEC, N).reshape(K // CB_VEC, N)
    codes = np.where(np.repeat(ok, group // CB_VEC, axis=0), codes, np.uint8(0))
    return CodebookLayer(K, N, group, codebook, codes.astype(np.uint8), scales)
