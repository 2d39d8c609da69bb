"""fp64 oracle: unpack -> eager dequantize -> plain dot product.

Test infrastructure only (see the package docstring).  Every function reads
the canonical layouts:

* uniform b-bit codes: ``uint32[K * b / 32, N]``, each column one little-endian
  bit stream with code k in bits ``[b*k, b*k + b)`` (for b = 2, 4, 8: word
  ``(j, n)`` bits ``[b*i, b*i + b)`` hold the code of weight ``(P*j + i, n)``,
  ``P = 32 / b``; 3-bit codes straddle words, 32 codes per 3 words);
* scales, zeros: fp16 ``[K / g, N]`` (zeros hold integers);
* LUT4 codes: ``uint8[K / 2, N]``, low nibble = even k; ``absmax`` fp32
  ``[K / 64, N]``; ``lut`` fp16 ``[16]``;
* Tile-COO: 128 x 128 (K x N) tiles numbered ``t = kt * (N / 128) + nt``,
  ``offsets[T + 1]`` (uint32), ``rc[nnz, 2]`` = (k - 128 kt, n - 128 nt) as
  uint8, ``vals[nnz]`` fp16.

Sources followed (page, section):

* asymmetric group dequantization ``w = s * (q - z)`` with per-group scale and
  zero: QFactory page, "问题与动机" (fine-grained asymmetric group-wise
  quantization with scale/zero auxiliary parameters) and observation 1
  (group size 128, asymmetric);
* the deferred-dequantization identity, whose weight-only case is
  ``sum_k x_k s (q_k - z) = s (sum_k q_k x_k - z sum_k x_k)``: QFactory page,
  observation 2 (J-matrix expansion of ``A_{z1} B_{z2}``, Table 2);
* table dequantization ``w = lut[q] * absmax``: "Fast NF4 Dequantization
  Kernels" page, abstract and method section (NF4 codes turned back into
  values through a 16-entry table);
* dense + sparse outlier decomposition ``y = x dequant(W_dense) + x W_out``:
  FlashQuant page, English abstract;
* codebook (vector) quantization, m = 1 codebook of 2^b centroids of length v,
  per-group normalization: ``w[k, n] = s[k // g, n] * C[code[k // v, n], k % v]``;
  and its Psumbook evaluation ``p[j, i] = sum_t C[i, t] x[v j + t]``,
  ``y[n] = sum_g s[g, n] sum_{j in g} p[j, code[j, n]]``: CodeGEMM page, method
  (overall framework, key designs one and four);
* stand-alone dequantization for prefill (fp16 weights written back to global
  memory, then an ordinary fp16 matmul): "Fast NF4 Dequantization Kernels"
  page, method section (technical framework: load codes, dequantize, write
  FP16 back for the following computation); QFactory page, assumption stress
  test and limitation 1 (prefill and large batches are compute-bound).

Parity status: every function here is pinned by tests that do not re-state
its formula (bounds against the unquantized weights, hand-derived golden
fixtures, exact-integer identities, brute force on tiny inputs); see the
``tests/test_oracle_*.py`` modules.  The comparison metric ``parity_errors``
is pinned by hand-computed cases and planted mistakes in
``tests/test_oracle_parity_metric.py``.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

TILE = 128


def _col_select(a: np.ndarray, cols: Optional[Sequence[int]]) -> np.ndarray:
    return a if cols is None else a[:, np.asarray(cols)]


# ---------------------------------------------------------------------------
# uniform asymmetric formats (W2 / W4 / W8)


def unpack_uniform(qweight: np.ndarray, bits: int, cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """Canonical words -> ``uint8[K, N]`` codes.  Each column's words form one little-endian
    bit stream (word j = stream bits 32 j .. 32 j + 31); code k is stream bits
    ``[bits*k, bits*k + bits)``.  For bits dividing 32 this reads ``P = 32 / bits`` whole
    codes per word; 3-bit codes may straddle two words."""
    words = _col_select(qweight, cols).astype(np.uint32)
    mask = np.uint32((1 << bits) - 1)
    W, N = words.shape
    if 32 % bits == 0:
        P = 32 // bits
        codes = np.empty((W * P, N), dtype=np.uint8)
        for i in range(P):
            codes[i::P, :] = (words >> np.uint32(bits * i)) & mask
        return codes
    K = W * 32 // bits
    w64 = words.astype(np.uint64)
    nxt = np.vstack([w64[1:], np.zeros((1, N), dtype=np.uint64)])
    pair = w64 | (nxt << np.uint64(32))        # stream bits 32 j .. 32 j + 63
    codes = np.empty((K, N), dtype=np.uint8)
    for k in range(K):
        o = bits * k
        codes[k] = (pair[o // 32] >> np.uint64(o % 32)) & np.uint64(mask)
    return codes


def dequant_uniform(codes: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
                    group: int, cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """Eager dequantization: ``w[k, n] = s[k // g, n] * (q[k, n] - z[k // g, n])`` in fp64."""
    s = _col_select(scales, cols).astype(np.float64)
    z = _col_select(zeros, cols).astype(np.float64)
    K = codes.shape[0]
    gidx = np.arange(K) // group
    return s[gidx, :] * (codes.astype(np.float64) - z[gidx, :])


def gemv_uniform(x: np.ndarray, qweight: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
                 bits: int, group: int, cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """``y[M, N] = x[M, K] @ dequant(W)[K, N]`` in fp64."""
    codes = unpack_uniform(qweight, bits, cols)
    w = dequant_uniform(codes, scales, zeros, group, cols)
    return x.astype(np.float64) @ w


# ---------------------------------------------------------------------------
# the two forms of the weight-only deferred-dequantization identity, in exact
# integer arithmetic.  fp16 x times 2^24 is an integer for every finite fp16
# value (normal or subnormal), so both forms are exact in int64 for K <= 2^14.


def x_as_integers(x: np.ndarray) -> np.ndarray:
    xi = x.astype(np.float64) * float(1 << 24)
    out = xi.astype(np.int64)
    assert np.array_equal(out.astype(np.float64), xi)
    return out


def eager_group_sums(x: np.ndarray, codes: np.ndarray, zeros: np.ndarray, group: int) -> np.ndarray:
    """``E[m, g, n] = sum_{k in g} (q[k, n] - z[g, n]) * X[m, k]`` (int64, X = 2^24 x)."""
    X = x_as_integers(x)
    M, K = X.shape
    N = codes.shape[1]
    G = K // group
    z = zeros.astype(np.int64)
    E = np.zeros((M, G, N), dtype=np.int64)
    for g in range(G):
        sl = slice(g * group, (g + 1) * group)
        E[:, g, :] = X[:, sl] @ (codes[sl].astype(np.int64) - z[g][None, :])
    return E


def deferred_group_sums(x: np.ndarray, codes: np.ndarray, zeros: np.ndarray, group: int) -> np.ndarray:
    """``D[m, g, n] = sum_{k in g} q[k, n] X[m, k] - z[g, n] * sum_{k in g} X[m, k]`` (int64)."""
    X = x_as_integers(x)
    M, K = X.shape
    N = codes.shape[1]
    G = K // group
    z = zeros.astype(np.int64)
    D = np.zeros((M, G, N), dtype=np.int64)
    for g in range(G):
        sl = slice(g * group, (g + 1) * group)
        dot = X[:, sl] @ codes[sl].astype(np.int64)
        xsum = X[:, sl].sum(axis=1)
        D[:, g, :] = dot - xsum[:, None] * z[g][None, :]
    return D


def gemv_from_group_sums(S: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """``y[m, n] = 2^-24 * sum_g s[g, n] * S[m, g, n]`` in fp64 (groups summed in order)."""
    s = scales.astype(np.float64)
    M, G, N = S.shape
    y = np.zeros((M, N), dtype=np.float64)
    for g in range(G):
        y += s[g][None, :] * S[:, g, :].astype(np.float64)
    return y * 2.0 ** -24


# ---------------------------------------------------------------------------
# LUT4 (NF4-style)


def unpack_lut4(qbytes: np.ndarray, cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """Canonical ``uint8[K / 2, N]`` -> ``uint8[K, N]`` codes (low nibble = even k)."""
    b = _col_select(qbytes, cols)
    K2, N = b.shape
    codes = np.empty((2 * K2, N), dtype=np.uint8)
    codes[0::2] = b & 0x0F
    codes[1::2] = b >> 4
    return codes


def dequant_lut4(codes: np.ndarray, lut: np.ndarray, absmax: np.ndarray, block: int,
                 cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """``w[k, n] = lut[q[k, n]] * absmax[k // block, n]`` in fp64 (the product is exact)."""
    a = _col_select(absmax, cols).astype(np.float64)
    table = lut.astype(np.float64)
    K = codes.shape[0]
    bidx = np.arange(K) // block
    return table[codes] * a[bidx, :]


def dequant_lut4_fp32(codes: np.ndarray, lut: np.ndarray, absmax: np.ndarray, block: int,
                      cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """The fp32 value of a dequantized LUT4 weight: the exact fp64 product rounded once to fp32."""
    return dequant_lut4(codes, lut, absmax, block, cols).astype(np.float32)


def gemv_lut4(x: np.ndarray, qbytes: np.ndarray, lut: np.ndarray, absmax: np.ndarray,
              block: int, cols: Optional[Sequence[int]] = None) -> np.ndarray:
    codes = unpack_lut4(qbytes, cols)
    return x.astype(np.float64) @ dequant_lut4(codes, lut, absmax, block, cols)


# ---------------------------------------------------------------------------
# outlier-aware W4: dense low-bit part + fp16 Tile-COO part


def tilecoo_to_dense(offsets: np.ndarray, rc: np.ndarray, vals: np.ndarray, K: int, N: int,
                     cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """Scatter the Tile-COO outliers into an fp64 ``[K, N]`` (or ``[K, len(cols)]``) matrix."""
    tiles_n = N // TILE
    T = (K // TILE) * tiles_n
    counts = np.diff(offsets.astype(np.int64))
    assert counts.shape[0] == T
    t = np.repeat(np.arange(T), counts)
    k = (t // tiles_n) * TILE + rc[:, 0].astype(np.int64)
    n = (t % tiles_n) * TILE + rc[:, 1].astype(np.int64)
    v = vals.astype(np.float64)
    if cols is None:
        out = np.zeros((K, N), dtype=np.float64)
        np.add.at(out, (k, n), v)
        return out
    cols = np.asarray(cols, dtype=np.int64)
    out = np.zeros((K, len(cols)), dtype=np.float64)
    pos = np.full(N, -1, dtype=np.int64)
    pos[cols] = np.arange(len(cols))
    keep = pos[n] >= 0
    np.add.at(out, (k[keep], pos[n[keep]]), v[keep])
    return out


def gemv_outlier(x: np.ndarray, qweight: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
                 offsets: np.ndarray, rc: np.ndarray, vals: np.ndarray, bits: int, group: int,
                 cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """``y = x @ dequant(W_dense) + x @ W_outlier`` in fp64."""
    K = x.shape[1]
    N = qweight.shape[1]
    dense = gemv_uniform(x, qweight, scales, zeros, bits, group, cols)
    sparse = x.astype(np.float64) @ tilecoo_to_dense(offsets, rc, vals, K, N, cols)
    return dense + sparse


# ---------------------------------------------------------------------------
# codebook quantization (CodeGEMM, m = 1): codes uint8 [K / v, N], codebook
# [2^b, v], scales [K / g, N]


def dequant_codebook(codes: np.ndarray, codebook: np.ndarray, scales: np.ndarray, v: int,
                     group: int, cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """``w[k, n] = s[k // g, n] * C[code[k // v, n], k % v]`` in fp64."""
    c = _col_select(codes, cols)
    s = _col_select(scales, cols).astype(np.float64)
    C = codebook.astype(np.float64)
    K = c.shape[0] * v
    k = np.arange(K)
    return s[k // group, :] * C[c[k // v, :], (k % v)[:, None]]


def gemv_codebook(x: np.ndarray, codes: np.ndarray, codebook: np.ndarray, scales: np.ndarray,
                  v: int, group: int, cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """``y = x @ dequant(W)`` in fp64."""
    return x.astype(np.float64) @ dequant_codebook(codes, codebook, scales, v, group, cols)


def psumbook(x: np.ndarray, codebook: np.ndarray, v: int) -> np.ndarray:
    """``P[m, j, i] = sum_t C[i, t] * x[m, v j + t]`` (fp64): every input slice of length v
    against every centroid."""
    xs = x.astype(np.float64)
    M, K = xs.shape
    return xs.reshape(M, K // v, v) @ codebook.astype(np.float64).T


def gemv_codebook_psumbook(x: np.ndarray, codes: np.ndarray, codebook: np.ndarray,
                           scales: np.ndarray, v: int, group: int,
                           cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """The Psumbook evaluation: build P, look each code up, sum per group, scale, sum groups."""
    P = psumbook(x, codebook, v)
    c = _col_select(codes, cols).astype(np.int64)
    s = _col_select(scales, cols).astype(np.float64)
    M = P.shape[0]
    J, N = c.shape
    per = group // v
    y = np.zeros((M, N), dtype=np.float64)
    for g in range(J // per):
        acc = np.zeros((M, N), dtype=np.float64)
        for j in range(g * per, (g + 1) * per):
            acc += P[:, j, :][:, c[j]]
        y += s[g][None, :] * acc
    return y


# ---------------------------------------------------------------------------
# stand-alone dequantization to fp16 + dense matmul (prefill, M >> 16)
#
# The fp16 weights are returned transposed, ``[N, K]`` (one row per output
# column, the layout of a linear layer's weight matrix).  Readings taken:
# a uniform weight is the exact ``s (q - z)`` rounded once to fp16 (round to
# nearest even); a LUT4 weight is the fp32 product ``lut[q] * absmax`` rounded
# to fp16, i.e. the fp32 dequantized value of the NF4 page's method (the
# codebook value times the block absmax in fp32) stored as FP16.


def dequant_uniform_fp16_nk(qweight: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
                            bits: int, group: int) -> np.ndarray:
    """fp16 ``[N, K]``: ``fp16(s[k // g, n] * (q[k, n] - z[k // g, n]))`` transposed."""
    w = dequant_uniform(unpack_uniform(qweight, bits), scales, zeros, group)
    return np.ascontiguousarray(w.T).astype(np.float16)


def dequant_lut4_fp16_nk(qbytes: np.ndarray, lut: np.ndarray, absmax: np.ndarray,
                         block: int) -> np.ndarray:
    """fp16 ``[N, K]``: ``fp16(fp32(lut[q[k, n]] * absmax[k // block, n]))`` transposed."""
    w32 = dequant_lut4_fp32(unpack_lut4(qbytes), lut, absmax, block)
    return np.ascontiguousarray(w32.T).astype(np.float16)


def prefill_matmul(x: np.ndarray, w16_nk: np.ndarray) -> np.ndarray:
    """``y[M, N] = x[M, K] @ W[N, K]^T`` in fp64 on the fp16 weights."""
    return x.astype(np.float64) @ w16_nk.astype(np.float64).T


# ---------------------------------------------------------------------------
# comparison metric shared by the parity tests


def parity_errors(y: np.ndarray, y_ref: np.ndarray):
    """(relative L2 error, max abs error / max |y_ref|) of ``y`` against ``y_ref``."""
    y = y.astype(np.float64)
    r = y_ref.astype(np.float64)
    den = np.linalg.norm(r)
    rel = float(np.linalg.norm(y - r) / den) if den > 0 else float(np.linalg.norm(y - r))
    mref = float(np.abs(r).max()) if r.size else 0.0
    mabs = float(np.abs(y - r).max()) if r.size else 0.0
    return rel, (mabs / mref if mref > 0 else mabs)
