// Fused dequant-GEMV kernels for sm_100a.
//
//   y[m, n] = sum_g s[g, n] ( sum_{k in g} q[k, n] x[m, k] - z[g, n] sum_{k in g} x[m, k] )
//
// the weight-only form of the deferred-dequantization identity (QFactory page,
// observation 2 / Table 2); the LUT4 variant sums absmax[b, n] * sum_{k in b} lut[q] x
// over 64-element blocks, and the outlier variant adds x . W_outlier from Tile-COO.
//
// Design (B200):
//  * Work units are (128-column block, 128-element group) pairs, split evenly over a
//    persistent grid of C CTAs (stream-K): CTA c owns the contiguous unit range
//    [c U / C, (c+1) U / C).  Every CTA streams one contiguous byte range of the
//    packed weights and the load balance is within one unit.  A range cuts at most
//    two blocks; their partial sums meet in an fp32 workspace and the last CTA to
//    arrive at a block (atomic counter, no waiting) adds them up in a fixed order.
//  * Each warp owns T 16-column tiles of the block.  A lane reads its 8 K-steps of a
//    tile-group with one 256-bit (W4, LUT4; two for W8) or 128-bit (W2) evict-first
//    load; weights are used once, so they skip L1 and leave L2 first.  Loads run D
//    groups ahead of the math.
//  * Codes become tensor-core operands with one AND each: a code in the low mantissa
//    bits of an fp16 with zero exponent is the exact subnormal q * 2^-24 (times a
//    power of two fixed by its bit field, undone in the epilogue).  The inner dot
//    sum_k q x runs on mma.sync m16n8k16 with fp32 accumulation; A is the weight tile
//    (16 columns x 16 K), B is x (8 rows per MMA).  That keeps the ALU work near
//    0.6 instructions per weight, which the 16-lane integer pipe of a sub-partition
//    sustains at HBM speed, where a CUDA-core convert-and-FMA path does not.
//  * sum_{k in g} x[m, k] comes from the same tensor core (an all-"one" A fragment
//    times the x fragment), once per group per warp, in the row scales of the codes.
//    The epilogue is two FMAs per output per group: acc += s * (d - z * xsum).
//  * LUT4 codes index a 256-entry table of fp16 pairs (one byte = the two codes of a
//    fragment register) replicated 32 times in shared memory, one copy per bank.
//  * The outlier variant adds the Tile-COO entries of each visited 128 x 128 tile into
//    a shared fp32 y tile while the dense part streams, reusing x lines the dense
//    path has just pulled into L1; the y tile joins the dense sums at the end of the
//    unit range, before the split-K fix-up.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "layout.h"

namespace qlk {

using namespace qlayout;

constexpr int kMaxOutlierGroups = 512;  // K <= 65536 for the outlier variant

struct GemvParams {
  const __half* x;            // [M][K]
  const uint8_t* qw;          // packed codes
  const __half* sc;           // packed scales (uniform) | lut16 (LUT4)
  const void* zp;             // packed zeros (fp16) | packed absmax (fp32)
  const uint32_t* tile_off;   // Tile-COO offsets, tiles in (block, group) order
  const uint16_t* tile_rc;    // row | col << 8
  const uint16_t* tile_val;   // fp16 bits
  __half* y;                  // [M][N]
  float* partials;            // split-K slots [2C][W][T][32][4 MT]
  uint32_t* counters;         // [nblocks][W]
  int M, N, K, G, nblocks, ntiles;
  long long U;                // nblocks * G
  int C;                      // CTAs
};

template <int FMT> struct Fmt;
template <> struct Fmt<kW4> {
  static constexpr int kWords = 8;
  static constexpr uint32_t kOnesHi = 0x00100010u;  // rows gi+8 carry a factor 16
  static constexpr float kHiScale = 1.0f / 16.0f;
};
template <> struct Fmt<kW2> {
  static constexpr int kWords = 4;
  static constexpr uint32_t kOnesHi = 0x00040004u;  // rows gi+8 carry a factor 4
  static constexpr float kHiScale = 1.0f / 4.0f;
};
template <> struct Fmt<kW8> {
  static constexpr int kWords = 16;
  static constexpr uint32_t kOnesHi = 0x00010001u;
  static constexpr float kHiScale = 1.0f;
};
template <> struct Fmt<kLUT4> {
  static constexpr int kWords = 8;
  static constexpr uint32_t kOnesHi = 0;
  static constexpr float kHiScale = 1.0f;
};

constexpr uint32_t kOnesLo = 0x00010001u;  // fp16 pair (2^-24, 2^-24)
constexpr float kTwo24 = 16777216.0f;

// ---------------------------------------------------------------------------
// memory access helpers

__device__ __forceinline__ void ldg_stream(const uint8_t* p, uint32_t (&r)[8]) {
  asm volatile(
      "ld.global.nc.L1::no_allocate.L2::evict_first.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "l"(p));
}

__device__ __forceinline__ void ldg_stream(const uint8_t* p, uint32_t (&r)[4], uint64_t pol) {
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "l"(p), "l"(pol));
}

__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

template <int FMT>
__device__ __forceinline__ void load_chunk(const uint8_t* p, uint32_t (&w)[Fmt<FMT>::kWords],
                                           uint64_t pol) {
  if constexpr (FMT == kW2) {
    ldg_stream(p, w, pol);
  } else if constexpr (FMT == kW8) {
    uint32_t a[8], b[8];
    ldg_stream(p, a);
    ldg_stream(p + 32, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[i] = a[i];
      w[8 + i] = b[i];
    }
  } else {
    ldg_stream(p, w);
  }
}

__device__ __forceinline__ uint4 ldg_x(const __half* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// ---------------------------------------------------------------------------
// tensor-core step: c[0..3] += A (16 x 16, fp16) * B (16 x 8, fp16), fp32 accumulate

__device__ __forceinline__ void hmma(float* c, const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment (a0a1, a2a3, a4a5, a6a7) of step s from a lane's words.  For the uniform
// formats each half holds code << shift, the shift fixed per register (layout.h):
// W4 rows gi+8 carry x16, W2 rows gi+8 carry x4 and odd steps x16.
template <int FMT>
__device__ __forceinline__ void frag_uniform(const uint32_t* w, int s, uint32_t (&a)[4]) {
  if constexpr (FMT == kW4) {
    const uint32_t v = w[s], h = v >> 8;
    a[0] = v & 0x000F000Fu;  // row gi,   dk 0 | dk 1
    a[1] = v & 0x00F000F0u;  // row gi+8, dk 0 | dk 1
    a[2] = h & 0x000F000Fu;  // row gi,   dk 2 | dk 3
    a[3] = h & 0x00F000F0u;  // row gi+8, dk 2 | dk 3
  } else if constexpr (FMT == kW2) {
    const uint32_t v = w[s >> 1], h = v >> 8;
    const uint32_t m0 = (s & 1) ? 0x00300030u : 0x00030003u;
    const uint32_t m1 = (s & 1) ? 0x00C000C0u : 0x000C000Cu;
    a[0] = v & m0;
    a[1] = v & m1;
    a[2] = h & m0;
    a[3] = h & m1;
  } else {  // W8
    const uint32_t v0 = w[2 * s], v1 = w[2 * s + 1];
    a[0] = v0 & 0x00FF00FFu;
    a[1] = v1 & 0x00FF00FFu;
    a[2] = (v0 >> 8) & 0x00FF00FFu;
    a[3] = (v1 >> 8) & 0x00FF00FFu;
  }
}

// LUT4: byte j of word s holds the two codes of fragment register j; the replicated
// table gives the fp16 pair (lut[lo], lut[hi]) from the lane's own bank.
__device__ __forceinline__ void frag_lut(uint32_t v, const uint32_t* tbl, int lane,
                                         uint32_t (&a)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) a[j] = tbl[(((v >> (8 * j)) & 0xFFu) << 5) | (uint32_t)lane];
}

__device__ __forceinline__ void build_lut_table(uint32_t* tbl, const __half* lut16, int tid,
                                                int nthreads) {
  for (int e = tid; e < 256 * 32; e += nthreads) {
    const int entry = e >> 5;
    const uint32_t lo = __half_as_ushort(lut16[entry & 15]);
    const uint32_t hi = __half_as_ushort(lut16[entry >> 4]);
    tbl[e] = lo | (hi << 16);
  }
}

// ---------------------------------------------------------------------------
// stream-K partition helpers

__host__ __device__ __forceinline__ long long unit_begin(long long c, long long U, long long C) {
  return c * U / C;
}
// CTA whose unit range contains unit u.
__host__ __device__ __forceinline__ int cta_of_unit(long long u, long long U, long long C) {
  return (int)(((u + 1) * C - 1) / U);
}

// ---------------------------------------------------------------------------

template <int FMT, int MT, int T, int W, int D, bool OUTL>
struct Gemv {
  static constexpr int KW = Fmt<FMT>::kWords;
  static constexpr int NACC = 4 * MT;  // accumulators per tile per lane
  static constexpr bool kLut = (FMT == kLUT4);
  static constexpr int kThreads = W * 32;

  struct Buf {
    uint32_t w[T][KW];
    uint32_t p0[T];   // scale pair (uniform)
    uint32_t p1[T];   // zero pair (uniform)
    float4 am[T];     // absmax (LUT4)
    uint4 xr[4];      // x fragment, rows gi (prefetched when MT == 1)
    uint32_t orc;     // this thread's outlier of the tile: row | col << 8
    uint32_t oval;    // its fp16 value
    uint32_t oend;    // end offset of the tile's entries
  };

  struct Smem {
    uint32_t lut[kLut ? 256 * 32 : 1];
    float ysm[OUTL ? 16 : 1][OUTL ? 128 : 1];
    uint32_t toff[OUTL ? kMaxOutlierGroups + 1 : 1];
  };

  __device__ static void load(const GemvParams& P, const Smem& sm, int b, int g, int ga, int tb,
                              int warp, int lane, uint64_t pol, Buf& buf) {
    const int gi = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int i = 0; i < T; ++i) {
      const int jj = warp * T + i;
      if (jj < tb) {
        const long long ch = chunk_index(b, g, jj, P.G, P.ntiles);
        load_chunk<FMT>(P.qw + ch * chunk_bytes(FMT) + lane * KW * 4, buf.w[i], pol);
        if constexpr (kLut) {
          buf.am[i] = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(P.zp) +
                                                            ch * 32 + gi * 4));
        } else {
          buf.p0[i] = __ldg(reinterpret_cast<const uint32_t*>(P.sc + ch * 16 + gi * 2));
          buf.p1[i] = __ldg(reinterpret_cast<const uint32_t*>(static_cast<const __half*>(P.zp) +
                                                              ch * 16 + gi * 2));
        }
      }
    }
    if constexpr (MT == 1) {
      if (gi < P.M && warp * T < tb) {
        const __half* xp = P.x + (size_t)gi * P.K + (size_t)g * kGroup + 8 * t4;
#pragma unroll
        for (int p = 0; p < 4; ++p) buf.xr[p] = ldg_x(xp + 32 * p);
      } else {
#pragma unroll
        for (int p = 0; p < 4; ++p) buf.xr[p] = make_uint4(0, 0, 0, 0);
      }
    }
    if constexpr (OUTL) {
      const uint32_t e = sm.toff[g - ga] + threadIdx.x;
      buf.oend = sm.toff[g - ga + 1];
      if (e < buf.oend) {
        buf.orc = __ldg(P.tile_rc + e);
        buf.oval = __ldg(P.tile_val + e);
      }
    }
  }

  // Dense work of one group of the warp's tiles: MMAs plus the group epilogue.
  __device__ static void compute(const GemvParams& P, const Smem& sm, int g, int tb, int warp,
                                 int lane, const Buf& buf, float (&acc)[T][NACC]) {
    const int gi = lane >> 2, t4 = lane & 3;
    uint4 xr[4], xr2[4];
    if constexpr (MT == 1) {
#pragma unroll
      for (int p = 0; p < 4; ++p) xr[p] = buf.xr[p];
    } else {
      const __half* xp = P.x + (size_t)gi * P.K + (size_t)g * kGroup + 8 * t4;
      const __half* xp2 = xp + (size_t)8 * P.K;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        xr[p] = gi < P.M ? ldg_x(xp + 32 * p) : make_uint4(0, 0, 0, 0);
        xr2[p] = gi + 8 < P.M ? ldg_x(xp2 + 32 * p) : make_uint4(0, 0, 0, 0);
      }
    }
    if constexpr (kLut) {
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        float c[T][NACC];
#pragma unroll
        for (int i = 0; i < T; ++i)
#pragma unroll
          for (int e = 0; e < NACC; ++e) c[i][e] = 0.f;
#pragma unroll
        for (int s = 4 * blk; s < 4 * blk + 4; ++s) {
          const int p = s >> 1, h = s & 1;
          const uint32_t b0 = h ? xr[p].z : xr[p].x, b1 = h ? xr[p].w : xr[p].y;
          uint32_t b2 = 0, b3 = 0;
          if constexpr (MT == 2) {
            b2 = h ? xr2[p].z : xr2[p].x;
            b3 = h ? xr2[p].w : xr2[p].y;
          }
#pragma unroll
          for (int i = 0; i < T; ++i) {
            uint32_t a[4];
            frag_lut(buf.w[i][s], sm.lut, lane, a);
            hmma(&c[i][0], a, b0, b1);
            if constexpr (MT == 2) hmma(&c[i][4], a, b2, b3);
          }
        }
#pragma unroll
        for (int i = 0; i < T; ++i) {
          if (warp * T + i < tb) {
            const float a0 = blk ? buf.am[i].z : buf.am[i].x;
            const float a8 = blk ? buf.am[i].w : buf.am[i].y;
#pragma unroll
            for (int e = 0; e < NACC; ++e) acc[i][e] = fmaf((e & 2) ? a8 : a0, c[i][e], acc[i][e]);
          }
        }
      }
    } else {
      const uint32_t kOnes[4] = {kOnesLo, Fmt<FMT>::kOnesHi, kOnesLo, Fmt<FMT>::kOnesHi};
      float cx[NACC];
      float c[T][NACC];
      float co[(FMT == kW2) ? T : 1][NACC];
#pragma unroll
      for (int e = 0; e < NACC; ++e) cx[e] = 0.f;
#pragma unroll
      for (int i = 0; i < T; ++i)
#pragma unroll
        for (int e = 0; e < NACC; ++e) {
          c[i][e] = 0.f;
          if constexpr (FMT == kW2) co[i][e] = 0.f;
        }
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int p = s >> 1, h = s & 1;
        const uint32_t b0 = h ? xr[p].z : xr[p].x, b1 = h ? xr[p].w : xr[p].y;
        uint32_t b2 = 0, b3 = 0;
        if constexpr (MT == 2) {
          b2 = h ? xr2[p].z : xr2[p].x;
          b3 = h ? xr2[p].w : xr2[p].y;
        }
        hmma(&cx[0], kOnes, b0, b1);
        if constexpr (MT == 2) hmma(&cx[4], kOnes, b2, b3);
#pragma unroll
        for (int i = 0; i < T; ++i) {
          uint32_t a[4];
          frag_uniform<FMT>(buf.w[i], s, a);
          if (FMT == kW2 && h == 1) {
            hmma(&co[i][0], a, b0, b1);
            if constexpr (MT == 2) hmma(&co[i][4], a, b2, b3);
          } else {
            hmma(&c[i][0], a, b0, b1);
            if constexpr (MT == 2) hmma(&c[i][4], a, b2, b3);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < T; ++i) {
        if (warp * T + i < tb) {
          const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&buf.p0[i]));
          const float2 z2 = __half22float2(*reinterpret_cast<const __half2*>(&buf.p1[i]));
#pragma unroll
          for (int e = 0; e < NACC; ++e) {
            float d = c[i][e];
            if constexpr (FMT == kW2) d = fmaf(co[i][e], 0.0625f, d);  // odd steps carry x16
            const float sc = (e & 2) ? s2.y : s2.x;
            const float zc = (e & 2) ? z2.y : z2.x;
            acc[i][e] = fmaf(sc, fmaf(-zc, cx[e], d), acc[i][e]);
          }
        }
      }
    }
  }

  // Outliers of tile (b, g): each thread takes entries threadIdx.x, +kThreads, ...
  __device__ static void outliers(const GemvParams& P, Smem& sm, int g, int ga, const Buf& buf) {
    const uint32_t e0 = sm.toff[g - ga] + threadIdx.x;
    for (uint32_t e = e0; e < buf.oend; e += kThreads) {
      const uint32_t rc = (e == e0) ? buf.orc : (uint32_t)__ldg(P.tile_rc + e);
      const uint32_t vb = (e == e0) ? buf.oval : (uint32_t)__ldg(P.tile_val + e);
      const int r = rc & 0xFF, col = rc >> 8;
      const float v = __half2float(__ushort_as_half((unsigned short)vb));
      const __half* xc = P.x + (size_t)g * kGroup + r;
      for (int m = 0; m < P.M; ++m) atomicAdd(&sm.ysm[m][col], v * __half2float(xc[(size_t)m * P.K]));
    }
  }

  __device__ static void store_y(const GemvParams& P, int b, int warp, int lane, int tb,
                                 const float (&v)[T][NACC]) {
    const int gi = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int i = 0; i < T; ++i) {
      const int jj = warp * T + i;
      if (jj >= tb) continue;
      const int nb = (b * kBlockTiles + jj) * kTileN + gi;
#pragma unroll
      for (int e = 0; e < NACC; ++e) {
        const int m = 2 * t4 + (e & 1) + 8 * (e >> 2);
        const int n = nb + ((e & 2) ? 8 : 0);
        if (m < P.M) P.y[(size_t)m * P.N + n] = __float2half_rn(v[i][e]);
      }
    }
  }

  __device__ static void segment(const GemvParams& P, Smem& sm, int b, int ga, int gb,
                                 int first_block, int warp, int lane, uint64_t pol) {
    const int tb = tiles_in_block(b, P.ntiles);
    float acc[T][NACC];
#pragma unroll
    for (int i = 0; i < T; ++i)
#pragma unroll
      for (int e = 0; e < NACC; ++e) acc[i][e] = 0.f;

    if constexpr (OUTL) {
      for (int i = threadIdx.x; i <= gb - ga; i += kThreads)
        sm.toff[i] = __ldg(P.tile_off + (long long)b * P.G + ga + i);
      __syncthreads();
    }

    Buf buf[D];
#pragma unroll
    for (int d = 0; d < D; ++d)
      if (ga + d < gb) load(P, sm, b, ga + d, ga, tb, warp, lane, pol, buf[d]);
    for (int g0 = ga; g0 < gb; g0 += D) {
#pragma unroll
      for (int d = 0; d < D; ++d) {
        const int g = g0 + d;
        if (g < gb) {
          if (warp * T < tb) compute(P, sm, g, tb, warp, lane, buf[d], acc);
          if constexpr (OUTL) outliers(P, sm, g, ga, buf[d]);
          if (g + D < gb) load(P, sm, b, g + D, ga, tb, warp, lane, pol, buf[d]);
        }
      }
    }

    // back to the true scale of y
    float v[T][NACC];
#pragma unroll
    for (int i = 0; i < T; ++i)
#pragma unroll
      for (int e = 0; e < NACC; ++e)
        v[i][e] = kLut ? acc[i][e] : acc[i][e] * ((e & 2) ? kTwo24 * Fmt<FMT>::kHiScale : kTwo24);

    if constexpr (OUTL) {
      __syncthreads();  // every thread's outliers of the range are in sm.ysm
      const int gi = lane >> 2, t4 = lane & 3;
#pragma unroll
      for (int i = 0; i < T; ++i) {
        const int jj = warp * T + i;
        if (jj >= tb) continue;
#pragma unroll
        for (int e = 0; e < NACC; ++e) {
          const int m = 2 * t4 + (e & 1) + 8 * (e >> 2);
          const int col = jj * kTileN + gi + ((e & 2) ? 8 : 0);
          if (m < P.M) {
            v[i][e] += sm.ysm[m][col];
            sm.ysm[m][col] = 0.f;
          }
        }
      }
      __syncthreads();  // cleared before the next range adds into it
    }

    if (warp * T >= tb) return;
    if (ga == 0 && gb == P.G) {  // this CTA owns the whole block
      store_y(P, b, warp, lane, tb, v);
      return;
    }
    // split-K fix-up
    const int c = blockIdx.x;
    const int slot = (b == first_block) ? 2 * c : 2 * c + 1;
    float* dst = P.partials + ((size_t)(slot * W + warp) * T * 32 + lane) * NACC;
#pragma unroll
    for (int i = 0; i < T; ++i)
#pragma unroll
      for (int e = 0; e < NACC; e += 4)
        *reinterpret_cast<float4*>(dst + (size_t)i * 32 * NACC + e) =
            make_float4(v[i][e], v[i][e + 1], v[i][e + 2], v[i][e + 3]);
    __threadfence();
    __syncwarp();
    uint32_t prev = 0;
    if (lane == 0) prev = atomicAdd(P.counters + (size_t)b * W + warp, 1u);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    const long long ub = (long long)b * P.G;
    const int cf = cta_of_unit(ub, P.U, P.C);
    const int cl = cta_of_unit(ub + P.G - 1, P.U, P.C);
    if (prev + 1 != (uint32_t)(cl - cf + 1)) return;
    __threadfence();
    float s[T][NACC];
#pragma unroll
    for (int i = 0; i < T; ++i)
#pragma unroll
      for (int e = 0; e < NACC; ++e) s[i][e] = 0.f;
    for (int cc = cf; cc <= cl; ++cc) {
      const int sl = (unit_begin(cc, P.U, P.C) >= ub) ? 2 * cc : 2 * cc + 1;
      const float* src = P.partials + ((size_t)(sl * W + warp) * T * 32 + lane) * NACC;
#pragma unroll
      for (int i = 0; i < T; ++i)
#pragma unroll
        for (int e = 0; e < NACC; e += 4) {
          const float4 q = __ldcg(reinterpret_cast<const float4*>(src + (size_t)i * 32 * NACC + e));
          s[i][e] += q.x;
          s[i][e + 1] += q.y;
          s[i][e + 2] += q.z;
          s[i][e + 3] += q.w;
        }
    }
    store_y(P, b, warp, lane, tb, s);
    if (lane == 0) P.counters[(size_t)b * W + warp] = 0u;  // ready for the next call
  }
};

template <int FMT, int MT, int T, int W, int D, bool OUTL>
__global__ void __launch_bounds__(W * 32) qgemv_kernel(const GemvParams P) {
  using G_ = Gemv<FMT, MT, T, W, D, OUTL>;
  __shared__ typename G_::Smem sm;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if constexpr (G_::kLut) {
    build_lut_table(sm.lut, P.sc, threadIdx.x, G_::kThreads);
  }
  if constexpr (OUTL) {
    for (int i = threadIdx.x; i < 16 * 128; i += G_::kThreads) (&sm.ysm[0][0])[i] = 0.f;
  }
  if constexpr (G_::kLut || OUTL) __syncthreads();
  const uint64_t pol = evict_first_policy();
  const long long u0 = unit_begin(blockIdx.x, P.U, P.C);
  const long long u1 = unit_begin(blockIdx.x + 1, P.U, P.C);
  const int first_block = (int)(u0 / P.G);
  for (long long u = u0; u < u1;) {
    const int b = (int)(u / P.G);
    const int ga = (int)(u - (long long)b * P.G);
    const long long be = (long long)(b + 1) * P.G;
    const long long ue = u1 < be ? u1 : be;
    const int gb = ga + (int)(ue - u);
    G_::segment(P, sm, b, ga, gb, first_block, warp, lane, pol);
    u = ue;
  }
}

}  // namespace qlk
