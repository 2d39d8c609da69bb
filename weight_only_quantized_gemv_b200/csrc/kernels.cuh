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
//    [c U / C, (c+1) U / C), i.e. one contiguous byte range of the packed weights.
//    A range cuts at most two blocks; their partial sums meet in an fp32 workspace
//    and the last CTA to arrive at a block (atomic counter, no waiting) adds them
//    up in a fixed order.
//  * One producer warp streams the range through a ring of S shared-memory stages
//    with plain bulk copies (cp.async.bulk, TMA 1-D, into its own CTA): per unit the codes of
//    the block's tiles, their scales/zeros (or absmax) and the M rows of x for the
//    group, all completing on the stage's mbarrier.  Weights and parameters carry
//    an L2 evict-first hint: they are read once.  Bytes in flight are bounded by
//    shared memory, not registers.
//  * Four consumer warps own two 16-column tiles each.  A consumer copies its part
//    of the stage into registers (conflict-free 128-bit reads), releases the stage
//    and does the math:
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
//  * The outlier variant adds the Tile-COO entries of each unit into a shared fp32
//    y tile, reading x from the same stage the dense path uses; the y tile joins
//    the dense sums at the end of the unit range, before the split-K fix-up.
//  * Every mbarrier wait is bounded.  A wait that runs out sets a bit in the workspace
//    error word and carries on, so a lost copy can corrupt results but never hang the
//    GPU.  Instances built for tests of the waits (TH) can shorten the limit, delay a
//    copy or hold a stage, and wait once more after flagging.
#pragma once
#include <cuda.h>  // CUtensorMap
#include <cuda_fp16.h>
#include <stdint.h>

#include "layout.h"

namespace qlk {

using namespace qlayout;

constexpr int kMaxUnitsPerCta = 1024;   // outlier variant: per-CTA offsets kept in smem
constexpr uint32_t kErrFullTimeout = 1u;
constexpr uint32_t kErrEmptyTimeout = 2u;
constexpr uint32_t kSpinLimit = 1u << 22;  // try_wait rounds before a wait is abandoned

struct GemvParams {
  const __half* x;            // [M][K]
  const uint8_t* qw;          // packed codes
  const __half* sc;           // packed scales (uniform) | lut16 (LUT4)
  const void* zp;             // packed zeros (fp16) | packed absmax (fp32)
  const uint32_t* tile_off;   // Tile-COO offsets, tiles in (block, group) order
  const uint16_t* tile_rc;    // row | col << 8
  const uint16_t* tile_val;   // fp16 bits
  __half* y;                  // [M][N]
  float* partials;            // split-K slots [2C][NC][T][32][4 MT]
  uint32_t* counters;         // [nblocks][NC]
  uint32_t* err;              // sticky error flags
  int M, N, K, G, nblocks, ntiles;
  int U;                      // nblocks * G
  int C;                      // CTAs
  uint32_t wait_limit;        // try_wait rounds before a wait is flagged (kSpinLimit)
  // tests of the bounded waits only (0 otherwise): bits 0-15 delay CTA 0's producer before
  // its first copy, bits 16-31 hold CTA 0's consumer warp 0 before it releases its first
  // stage, in microseconds
  uint32_t test_us;
};

template <int FMT> struct Fmt;
template <> struct Fmt<kW4> {
  static constexpr int kWords = 8;
  static constexpr uint32_t kOnesHi = 0x00100010u;  // rows gi+8 carry a factor 16
  static constexpr float kHiScale = 1.0f / 16.0f;
  static constexpr int kStagesPerWarpM8 = 1;
};
template <> struct Fmt<kW2> {
  static constexpr int kWords = 4;
  static constexpr uint32_t kOnesHi = 0x00040004u;  // rows gi+8 carry a factor 4
  static constexpr float kHiScale = 1.0f / 4.0f;
  static constexpr int kStagesPerWarpM8 = 2;
};
template <> struct Fmt<kW3> {  // low two bits as W2 codes (words 0..3), high bit in words 4, 5
  static constexpr int kWords = 6;
  static constexpr uint32_t kOnesHi = 0x00040004u;  // rows gi+8 carry a factor 4 (as W2)
  static constexpr float kHiScale = 1.0f / 4.0f;
  static constexpr int kStagesPerWarpM8 = 2;
};
template <> struct Fmt<kW8> {
  static constexpr int kWords = 16;
  static constexpr uint32_t kOnesHi = 0x00010001u;
  static constexpr float kHiScale = 1.0f;
  static constexpr int kStagesPerWarpM8 = 1;
};
template <> struct Fmt<kCB> {  // 8-bit codebook indices, two per step (rows gi, gi + 8)
  static constexpr int kWords = 4;
  static constexpr uint32_t kOnesHi = 0;
  static constexpr float kHiScale = 1.0f;
  static constexpr int kStagesPerWarpM8 = 1;  // with the 32 KB table: three CTAs per SM
};
template <> struct Fmt<kLUT4> {
  static constexpr int kWords = 8;
  static constexpr uint32_t kOnesHi = 0;
  static constexpr float kHiScale = 1.0f;
  static constexpr int kStagesPerWarpM8 = 1;
};

constexpr uint32_t kOnesLo = 0x00010001u;  // fp16 pair (2^-24, 2^-24)
constexpr float kTwo24 = 16777216.0f;

__host__ __device__ constexpr int align_to(int v, int a) { return (v + a - 1) / a * a; }

// Warps that share each unit by default: one for 4-bit codes at M <= 8 (the least work per
// unit), else a pair.  The host may pick more for layers too small to keep every warp busy.
__host__ __device__ constexpr int default_wpu(int fmt, int mt) { return (mt == 1 && fmt == kW4) ? 1 : 2; }

// Shared-memory layout of one kernel instance.  WPU warps share each unit, warp h of a group
// taking tiles (8 / WPU) h .. (8 / WPU) (h + 1) - 1.  M1: exactly one row of x (only the
// accumulator entries of batch column 0 are kept; x arrives by a 1-D bulk copy).  Every
// other instance serves M >= 2 and copies x as one 2-D tile per unit through a tensor map.
template <int FMT, int MT, bool OUTL, int WPU_, bool M1_ = false, int OCC_ = 0, int NS_ = 1>
struct Cfg {
  static constexpr bool M1 = M1_;
  // quantization sub-groups per 128-k unit (group size 128 / NS): W2 / W4 / W8 only.  Each
  // sub-group covers 8 / NS consecutive tensor-core steps (steps 2p, 2p + 1 hold k
  // 32 p .. 32 p + 31), so its scale and zero pairs stay in registers for those steps.
  static constexpr int NS = NS_;
  static_assert(NS == 1 || NS == 2 || NS == 4, "group 128, 64 or 32");
  static_assert(NS == 1 || (FMT != kLUT4 && FMT != kW3 && !OUTL && WPU_ == 2),
                "finer groups: W2 / W4 / W8, 2 warps per unit");
  static_assert(!M1 || MT == 1, "one row of x is the M <= 8 bucket");
  static constexpr int NC = 4;                       // consumer warps
  static constexpr int WPU = WPU_;
  static_assert(WPU == 1 || WPU == 2 || WPU == 4, "1, 2 or 4 warps per unit");
  static constexpr int NP = NC / WPU;                // warp groups, each takes whole units
  static constexpr int kTW = kBlockTiles / WPU;      // tiles of a unit per warp
  // tiles a warp holds in registers at once (independent accumulator chains)
  static constexpr int kQ = kTW < 4 ? kTW : (MT == 2 || FMT == kW8 || FMT == kW3 || NS > 1) ? 2 : 4;
  static constexpr int T = 2;                        // tiles per warp in the block epilogue
  static constexpr int kThreads = (NC + 1) * 32;     // + one producer warp
  static constexpr int KW = Fmt<FMT>::kWords;
  static constexpr int NACC = 4 * MT;
  // stages: warp group p uses the stages s = p (mod NP); one per warp at M <= 8 (two for
  // 2-bit codes, whose stages are small), two per group at M > 8
  static constexpr int S = NC * (MT == 1 ? Fmt<FMT>::kStagesPerWarpM8 : (WPU == 1 ? 2 : 1));
  // CTAs per SM the registers are sized for: OCC_, else the format's default (more CTAs,
  // fewer registers per thread)
  static constexpr int kOcc = OCC_;
  static constexpr int kMinCtas =
      OCC_ ? OCC_ : (FMT == kLUT4) ? 2 : (MT == 1 && FMT != kW8) ? 3 : 2;
  static constexpr int kChunkBytes = 128 * KW;
  static constexpr int kCodeBytes = kBlockTiles * kChunkBytes;
  static constexpr int kParamChunk = (FMT == kLUT4) ? 128 : 32 * NS;   // per tile, per array
  static constexpr int kParamBytes = (FMT == kLUT4) ? 8 * 128 : (FMT == kCB) ? 8 * 32 : 2 * 8 * 32 * NS;
  static constexpr int kZeroOff = 8 * 32 * NS;   // zeros after the 8 tiles' scales
  // x rows in a stage: the 2-D tile copy (M >= 2) writes them densely; the single-row
  // kernel keeps 16 bytes of padding, which spreads the fragment loads over the banks
  static constexpr int kXStride = M1 ? 272 : 256;
  static constexpr int kXRows = 8 * MT;
  static constexpr int kXOff = kCodeBytes + kParamBytes;
  static constexpr int kStageBytes = align_to(kXOff + kXRows * kXStride, 128);
  static constexpr int kRingBytes = S * kStageBytes;
  static constexpr int kBarOff = kRingBytes;                       // full[S], empty[S]
  static constexpr int kLutOff = align_to(kBarOff + 16 * S, 128);
  // LUT4: 256 fp16 pairs x 32 copies; CB: the 256 fp16 4-vectors x 16 copies
  static constexpr int kLutBytes = (FMT == kLUT4) ? 256 * 32 * 4 : (FMT == kCB) ? 256 * 16 * 8 : 0;
  static constexpr int kRedOff = kLutOff + kLutBytes;              // per-warp block sums
  // each warp holds kTW tiles.  The W4 M <= 8 variants (1, 2 or 4 warps per unit) all size
  // it for kTW = 8, so that they ask for the same shared memory: consecutive launches of
  // different variants then share one L1 / shared-memory split and overlap.
  static constexpr int kRedBytes =
      NC * ((FMT == kW4 && MT == 1) ? kBlockTiles : kTW) * 32 * NACC * 4;
  static constexpr int kYsmOff = kRedOff + kRedBytes;
  static constexpr int kYsmBytes = OUTL ? 16 * 128 * 4 : 0;
  static constexpr int kToffOff = kYsmOff + kYsmBytes;
  static constexpr int kToffBytes = OUTL ? (kMaxUnitsPerCta + 1) * 4 : 0;
  static constexpr int kSmemBytes = kToffOff + kToffBytes;
};

// ---------------------------------------------------------------------------
// PTX helpers: mbarriers, bulk copies, shared loads

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait for the phase with parity `parity` to complete; false if abandoned.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t limit) {
  for (uint32_t it = 0; it < limit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// Wait for a stage's phase, bounded by kSpinLimit rounds; a wait that gives up sets `bit` in
// the error word and carries on (the results are then undefined).  TH: the instances built
// for tests of the bounded waits, where the limit is P.wait_limit and a wait that passes it
// sets the flag and then waits at most kSpinLimit more rounds, so that a late copy still
// lands before it is read.  (Kept out of the other instances: in the unit loop the longer
// form costs the single-row kernel about 6 %.)
template <bool TH>
__device__ __forceinline__ void stage_wait(const GemvParams& P, uint32_t bar, uint32_t parity,
                                           uint32_t bit) {
  if constexpr (TH) {
    if (!mbar_wait(bar, parity, P.wait_limit)) {
      atomicOr(P.err, bit);
      mbar_wait(bar, parity, kSpinLimit);
    }
  } else {
    if (!mbar_wait(bar, parity, kSpinLimit)) atomicOr(P.err, bit);
  }
}

// Tests of the bounded waits: let `us` microseconds pass (a fixed, bounded delay).
__device__ __forceinline__ void test_delay(uint32_t us) {
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (;;) {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 >= 1000ull * us) return;
    __nanosleep(1000);
  }
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint16_t lds16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}

// Split-K arrival: atomic add at GPU scope with acquire-release semantics, returns the old value.
__device__ __forceinline__ uint32_t arrive_acq_rel(uint32_t* counter) {
  uint32_t old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(old) : "l"(counter) : "memory");
  return old;
}

__device__ __forceinline__ float4 ld_relaxed_gpu(const float4* p) {
  float4 v;
  asm volatile("ld.relaxed.gpu.global.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

// Programmatic dependent launch: let the next kernel in the stream start (it still waits
// for this grid to complete before it reads anything this grid wrote) / wait until the
// previous kernel in the stream has completed and its writes are visible.
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void consumer_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// tensor-core step: c[0..3] += A (16 x 16, fp16) * B (16 x 8, fp16), fp32 accumulate

__device__ __forceinline__ void hmma(float* c, const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// c[0..3] = A * B (the accumulator input is zero)
__device__ __forceinline__ void hmma0(float* c, const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// A fragment (a0a1, a2a3, a4a5, a6a7) of step s from a lane's words.  For the uniform
// formats each half holds code << shift, the shift fixed per register (layout.h):
// W4 rows gi+8 carry x16, W2 rows gi+8 carry x4 and odd steps x16.
__device__ __forceinline__ uint32_t shr8(uint32_t v) { return v >> 8; }

template <int FMT>
__device__ __forceinline__ void frag_uniform(const uint32_t* w, int s, uint32_t (&a)[4]) {
  if constexpr (FMT == kW4) {
    const uint32_t v = w[s], h = shr8(v);
    a[0] = v & 0x000F000Fu;  // row gi,   dk 0 | dk 1
    a[1] = v & 0x00F000F0u;  // row gi+8, dk 0 | dk 1
    a[2] = h & 0x000F000Fu;  // row gi,   dk 2 | dk 3
    a[3] = h & 0x00F000F0u;  // row gi+8, dk 2 | dk 3
  } else if constexpr (FMT == kW2) {
    const uint32_t v = w[s >> 1], h = shr8(v);
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
    a[2] = shr8(v0) & 0x00FF00FFu;
    a[3] = shr8(v1) & 0x00FF00FFu;
  }
}

// LUT4: byte j of word s holds the two codes of fragment register j; the replicated
// table gives the fp16 pair (lut[lo], lut[hi]) from the lane's own bank.
// tbl_lane = table base + 4 lane.  Entry (byte, lane) sits at byte * 128 + 4 lane: the byte
// comes out with one byte permute (ALU) and the address with one multiply-add (FMA pipe).
__device__ __forceinline__ void frag_lut(uint32_t v, uint32_t tbl_lane, uint32_t (&a)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t byte;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(byte) : "r"(v), "r"(0x4440u | (uint32_t)j));
    a[j] = lds32(byte * 128u + tbl_lane);
  }
}

// CB: entry (code, copy) at (16 code + copy) * 8 bytes, 16 copies of each 8-byte 4-vector;
// lane l reads copy l % 16, so the two 16-lane halves of a 64-bit load each touch all 32
// banks once.
__device__ __forceinline__ void build_cb_table(uint2* tbl, const __half* codebook, int tid,
                                               int nthreads) {
  const uint2* cb = reinterpret_cast<const uint2*>(codebook);
  for (int e = tid; e < 256 * 16; e += nthreads) tbl[e] = cb[e >> 4];
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

// 32-bit arithmetic: the host guarantees U * C < 2^31.
__host__ __device__ __forceinline__ int unit_begin(int c, int U, int C) {
  return (int)((unsigned)c * (unsigned)U / (unsigned)C);
}
// CTA whose unit range contains unit u.
__host__ __device__ __forceinline__ int cta_of_unit(int u, int U, int C) {
  return (int)(((unsigned)(u + 1) * (unsigned)C - 1u) / (unsigned)U);
}

// ---------------------------------------------------------------------------

template <int FMT, int MT, bool OUTL, int WPU_, bool M1_ = false, int OCC_ = 0, int NS_ = 1,
          bool TH = false>
struct Gemv {
  using C_ = Cfg<FMT, MT, OUTL, WPU_, M1_, OCC_, NS_>;
  static constexpr int NS = C_::NS;
  static constexpr int NC = C_::NC, T = C_::T, KW = C_::KW, NACC = C_::NACC, S = C_::S;
  static constexpr int WPU = C_::WPU, NP = C_::NP, kTW = C_::kTW;
  static constexpr bool kLut = (FMT == kLUT4);
  static constexpr bool kCb = (FMT == kCB);
  static constexpr int kBT = kBlockTiles;

  // x fragments of one unit (rows gi and, for MT == 2, gi + 8), from the stage.
  __device__ static void read_x(const GemvParams& P, uint32_t st, int lane, uint4 (&xr)[4],
                                uint4 (&xr2)[4]) {
    const int gi = lane >> 2, t4 = lane & 3;
    const uint32_t xb = st + C_::kXOff + gi * C_::kXStride + 16 * t4;
#pragma unroll
    for (int p = 0; p < 4; ++p) {  // rows >= M hold zeros (filled once at kernel start)
      xr[p] = lds128(xb + 64 * p);
      if constexpr (MT == 2) xr2[p] = lds128(xb + 8 * C_::kXStride + 64 * p);
    }
  }

  // The stage bytes of kQ tiles (j0 .. j0 + kQ - 1) of one unit, in registers.
  static constexpr int kQ = C_::kQ;
  struct Quad {
    uint32_t w[kQ][KW];
    uint32_t p0[kQ], p1[kQ];  // scale / zero pairs (uniform)
    float4 am[kQ];            // absmax (LUT4)
  };

  __device__ static void load_quad(uint32_t st, int j0, int lane, Quad& r) {
    const int gi = lane >> 2;
#pragma unroll
    for (int i = 0; i < kQ; ++i) {
      const uint32_t cb = st + (j0 + i) * C_::kChunkBytes + lane * 16;
#pragma unroll
      for (int q = 0; q < KW / 4; ++q) {
        const uint4 v = lds128(cb + q * 512);
        r.w[i][4 * q + 0] = v.x;
        r.w[i][4 * q + 1] = v.y;
        r.w[i][4 * q + 2] = v.z;
        r.w[i][4 * q + 3] = v.w;
      }
      if constexpr (FMT == kW3) {  // the high-bit plane: 8 bytes per lane after the quads
        const uint2 v = lds64(st + (j0 + i) * C_::kChunkBytes + 512 + lane * 8);
        r.w[i][4] = v.x;
        r.w[i][5] = v.y;
      }
      if constexpr (kLut) {
        const uint4 a = lds128(st + C_::kCodeBytes + (j0 + i) * 128 + gi * 16);
        r.am[i] = make_float4(__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z),
                              __uint_as_float(a.w));
      } else {
        r.p0[i] = lds32(st + C_::kCodeBytes + (j0 + i) * 32 + gi * 4);
        if constexpr (!kCb) r.p1[i] = lds32(st + C_::kCodeBytes + 256 + (j0 + i) * 32 + gi * 4);
      }
    }
  }

  // MMAs and group epilogue of kQ tiles: kQ independent accumulator chains per step.
  __device__ static void compute_quad(const Quad& r, int lane, uint32_t lut,
                                      const uint4 (&xr)[4], const uint4 (&xr2)[4],
                                      const float (&cx)[NACC], float (*acc)[NACC]) {
    const auto& w = r.w;
    if constexpr (kLut) {
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        float c[kQ][NACC];
#pragma unroll
        for (int s = 4 * blk; s < 4 * blk + 4; ++s) {
          const int p = s >> 1, h = s & 1;
          const uint32_t b0 = h ? xr[p].z : xr[p].x, b1 = h ? xr[p].w : xr[p].y;
#pragma unroll
          for (int i = 0; i < kQ; ++i) {
            uint32_t a[4];
            frag_lut(w[i][s], lut + 4u * (uint32_t)lane, a);
            const uint32_t b2 = h ? xr2[p].z : xr2[p].x, b3 = h ? xr2[p].w : xr2[p].y;
            if (s == 4 * blk) {
              hmma0(&c[i][0], a, b0, b1);
              if constexpr (MT == 2) hmma0(&c[i][4], a, b2, b3);
            } else {
              hmma(&c[i][0], a, b0, b1);
              if constexpr (MT == 2) hmma(&c[i][4], a, b2, b3);
            }
          }
        }
#pragma unroll
        for (int i = 0; i < kQ; ++i) {
          const float a0 = blk ? r.am[i].z : r.am[i].x;
          const float a8 = blk ? r.am[i].w : r.am[i].y;
#pragma unroll
          for (int e = 0; e < NACC; ++e)
            if (!C_::M1 || !(e & 1)) acc[i][e] = fmaf((e & 2) ? a8 : a0, c[i][e], acc[i][e]);
        }
      }
    } else if constexpr (kCb) {
      // Codebook: in step s the lane's fragment covers the 4 consecutive k of one codebook
      // vector for row gi (a0, a2) and one for row gi + 8 (a1, a3) (the fragments' k order
      // is the one x is staged in: real k = 32 (s / 2) + 8 t + 4 (s % 2) + 0..3).  Byte
      // 2 s + r8 of the lane's 16 code bytes indexes the vector; one 64-bit lookup in the
      // lane's copy of the table gives both registers of a row.
      const uint32_t tl = lut + 8u * (uint32_t)(lane & 15);
      float c[kQ][NACC];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int p = s >> 1, h = s & 1;
        const uint32_t b0 = h ? xr[p].z : xr[p].x, b1 = h ? xr[p].w : xr[p].y;
        uint32_t b2 = 0, b3 = 0;
        if constexpr (MT == 2) {
          b2 = h ? xr2[p].z : xr2[p].x;
          b3 = h ? xr2[p].w : xr2[p].y;
        }
#pragma unroll
        for (int i = 0; i < kQ; ++i) {
          const uint32_t v = w[i][s >> 1];
          uint32_t c0, c1;
          asm("prmt.b32 %0, %1, 0, %2;" : "=r"(c0) : "r"(v), "r"(0x4440u | (uint32_t)(2 * h)));
          asm("prmt.b32 %0, %1, 0, %2;" : "=r"(c1) : "r"(v), "r"(0x4440u | (uint32_t)(2 * h + 1)));
          const uint2 r0 = lds64(c0 * 128u + tl), r1 = lds64(c1 * 128u + tl);
          const uint32_t a[4] = {r0.x, r1.x, r0.y, r1.y};
          if (s == 0) {
            hmma0(&c[i][0], a, b0, b1);
            if constexpr (MT == 2) hmma0(&c[i][4], a, b2, b3);
          } else {
            hmma(&c[i][0], a, b0, b1);
            if constexpr (MT == 2) hmma(&c[i][4], a, b2, b3);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kQ; ++i) {
        const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&r.p0[i]));
#pragma unroll
        for (int e = 0; e < NACC; ++e) {
          if (C_::M1 && (e & 1)) continue;  // batch column 1 of the fragment: no such row
          acc[i][e] = fmaf((e & 2) ? s2.y : s2.x, c[i][e], acc[i][e]);
        }
      }
    } else if constexpr (FMT == kW3) {
      // W3 = W2 plane (even steps in c, odd steps, which carry x16, in co) + 4 x high-bit
      // plane (c1, every field at bit 0 of its half)
      float c[kQ][NACC], co[kQ][NACC], c1[kQ][NACC];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int p = s >> 1, h = s & 1;
        const uint32_t b0 = h ? xr[p].z : xr[p].x, b1 = h ? xr[p].w : xr[p].y;
        uint32_t b2 = 0, b3 = 0;
        if constexpr (MT == 2) {
          b2 = h ? xr2[p].z : xr2[p].x;
          b3 = h ? xr2[p].w : xr2[p].y;
        }
#pragma unroll
        for (int i = 0; i < kQ; ++i) {
          uint32_t a[4], a1[4];
          frag_uniform<kW2>(w[i], s, a);
          const uint32_t v1 = w[i][4 + (s >> 2)];
#pragma unroll
          for (int rr = 0; rr < 4; ++rr) a1[rr] = (v1 >> (4 * (s & 3) + rr)) & 0x00010001u;
          float* cs = h ? &co[i][0] : &c[i][0];
          if (s <= 1) {
            hmma0(cs, a, b0, b1);
            if constexpr (MT == 2) hmma0(cs + 4, a, b2, b3);
          } else {
            hmma(cs, a, b0, b1);
            if constexpr (MT == 2) hmma(cs + 4, a, b2, b3);
          }
          if (s == 0) {
            hmma0(&c1[i][0], a1, b0, b1);
            if constexpr (MT == 2) hmma0(&c1[i][4], a1, b2, b3);
          } else {
            hmma(&c1[i][0], a1, b0, b1);
            if constexpr (MT == 2) hmma(&c1[i][4], a1, b2, b3);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kQ; ++i) {
        const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&r.p0[i]));
        const float2 z2 = __half22float2(*reinterpret_cast<const __half2*>(&r.p1[i]));
#pragma unroll
        for (int e = 0; e < NACC; ++e) {
          if (C_::M1 && (e & 1)) continue;  // batch column 1 of the fragment: no such row
          // rows gi + 8 (e & 2) carry x4 in the W2 plane: their high bit weighs 4 x 4
          float d = fmaf(co[i][e], 0.0625f, c[i][e]);
          d = fmaf(c1[i][e], (e & 2) ? 16.0f : 4.0f, d);
          const float sc = (e & 2) ? s2.y : s2.x;
          const float zc = (e & 2) ? z2.y : z2.x;
          acc[i][e] = fmaf(sc, fmaf(-zc, cx[e], d), acc[i][e]);
        }
      }
    } else {
      float c[kQ][NACC];
      float co[(FMT == kW2) ? kQ : 1][NACC];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int p = s >> 1, h = s & 1;
        const uint32_t b0 = h ? xr[p].z : xr[p].x, b1 = h ? xr[p].w : xr[p].y;
        uint32_t b2 = 0, b3 = 0;
        if constexpr (MT == 2) {
          b2 = h ? xr2[p].z : xr2[p].x;
          b3 = h ? xr2[p].w : xr2[p].y;
        }
#pragma unroll
        for (int i = 0; i < kQ; ++i) {
          uint32_t a[4];
          frag_uniform<FMT>(w[i], s, a);
          if constexpr (FMT == kW2) {
            if (h == 1) {  // odd steps accumulate separately (their codes carry x16)
              if (s == 1) {
                hmma0(&co[i][0], a, b0, b1);
                if constexpr (MT == 2) hmma0(&co[i][4], a, b2, b3);
              } else {
                hmma(&co[i][0], a, b0, b1);
                if constexpr (MT == 2) hmma(&co[i][4], a, b2, b3);
              }
              continue;
            }
          }
          if (s == 0) {
            hmma0(&c[i][0], a, b0, b1);
            if constexpr (MT == 2) hmma0(&c[i][4], a, b2, b3);
          } else {
            hmma(&c[i][0], a, b0, b1);
            if constexpr (MT == 2) hmma(&c[i][4], a, b2, b3);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kQ; ++i) {
        const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&r.p0[i]));
        const float2 z2 = __half22float2(*reinterpret_cast<const __half2*>(&r.p1[i]));
#pragma unroll
        for (int e = 0; e < NACC; ++e) {
          if (C_::M1 && (e & 1)) continue;  // batch column 1 of the fragment: no such row
          float d = c[i][e];
          if constexpr (FMT == kW2) d = fmaf(co[i][e], 0.0625f, d);  // odd steps carry x16
          const float sc = (e & 2) ? s2.y : s2.x;
          const float zc = (e & 2) ? z2.y : z2.x;
          acc[i][e] = fmaf(sc, fmaf(-zc, cx[e], d), acc[i][e]);
        }
      }
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

  // End of a run of units of block b: combine the warps' sums (each warp then owns
  // tiles 2w, 2w+1), rescale, add outliers, write y or join the split-K fix-up.
  __device__ static void finish_block(const GemvParams& P, uint8_t* smem, int b, bool whole,
                                      int first_block, int warp, int lane,
                                      float (&acc)[kTW][NACC]) {
    const int tb = tiles_in_block(b, P.ntiles);
    float* red = reinterpret_cast<float*>(smem + C_::kRedOff);
    float* ysm = reinterpret_cast<float*>(smem + C_::kYsmOff);
    consumer_sync(NC * 32);  // all units of the run are done (and their outliers in ysm)
#pragma unroll
    for (int j = 0; j < kTW; ++j) {
#pragma unroll
      for (int e = 0; e < NACC; e += 4)
        *reinterpret_cast<float4*>(red + ((warp * kTW + j) * 32 + lane) * NACC + e) =
            make_float4(acc[j][e], acc[j][e + 1], acc[j][e + 2], acc[j][e + 3]);
#pragma unroll
      for (int e = 0; e < NACC; ++e) acc[j][e] = 0.f;
    }
    consumer_sync(NC * 32);
    // tile jj sits, in each warp group p, with warp WPU p + jj / kTW in slot jj % kTW
    float v[T][NACC];
#pragma unroll
    for (int i = 0; i < T; ++i) {
      const int jj = warp * T + i;
#pragma unroll
      for (int e = 0; e < NACC; ++e) v[i][e] = 0.f;
#pragma unroll
      for (int p2 = 0; p2 < NP; ++p2)
#pragma unroll
        for (int e = 0; e < NACC; e += 4) {
          const int w2 = WPU * p2 + jj / kTW;
          const float4 q =
              *reinterpret_cast<const float4*>(red + ((w2 * kTW + jj % kTW) * 32 + lane) * NACC + e);
          v[i][e] += q.x;
          v[i][e + 1] += q.y;
          v[i][e + 2] += q.z;
          v[i][e + 3] += q.w;
        }
#pragma unroll
      for (int e = 0; e < NACC; ++e)
        if (!kLut && !kCb) v[i][e] *= (e & 2) ? kTwo24 * Fmt<FMT>::kHiScale : kTwo24;
    }
    if constexpr (OUTL) {  // the outlier sums of this warp's tiles, then cleared
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
            v[i][e] += ysm[m * 128 + col];
            ysm[m * 128 + col] = 0.f;
          }
        }
      }
      // the next run's units add into the tile only after every warp has read and cleared
      // its part (a warp that went on early would add into sums another warp still reads)
      consumer_sync(NC * 32);
    }
    if (warp * T >= tb) return;
    if (whole) {
      store_y(P, b, warp, lane, tb, v);
      return;
    }
    // split-K fix-up: publish this CTA's partial, the last contributor sums them all
    const int c = blockIdx.x;
    const int slot = (b == first_block) ? 2 * c : 2 * c + 1;
    float* dst = P.partials + ((size_t)(slot * NC + warp) * T * 32 + lane) * NACC;
#pragma unroll
    for (int i = 0; i < T; ++i)
#pragma unroll
      for (int e = 0; e < NACC; e += 4)
        *reinterpret_cast<float4*>(dst + (size_t)i * 32 * NACC + e) =
            make_float4(v[i][e], v[i][e + 1], v[i][e + 2], v[i][e + 3]);
    // the warp's stores, then one acquire-release arrival: it publishes them (release) and,
    // for the last contributor, makes every other contributor's partial visible (acquire)
    __syncwarp();
    uint32_t prev = 0;
    if (lane == 0) prev = arrive_acq_rel(P.counters + (size_t)b * NC + warp);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    const int ub = b * P.G;
    const int cf = cta_of_unit(ub, P.U, P.C);
    const int cl = cta_of_unit(ub + P.G - 1, P.U, P.C);
    if (prev + 1 != (uint32_t)(cl - cf + 1)) return;
    __syncwarp();
    float s[T][NACC];
#pragma unroll
    for (int i = 0; i < T; ++i)
#pragma unroll
      for (int e = 0; e < NACC; ++e) s[i][e] = 0.f;
    // contributors in CTA order; loads of up to kF slots are in flight at once.  One at a
    // time, except in the small-layer variant: the registers of a deeper batch, though only
    // live here, cost the main loop more spills than the shallower fix-up costs, and only
    // small layers (many contributors per block, little work) feel the fix-up's latency.
    constexpr int kF = C_::kOcc == 2 ? 4 : 1;
    for (int c0 = cf; c0 <= cl; c0 += kF) {
      float4 q[kF][T][NACC / 4];
#pragma unroll
      for (int f = 0; f < kF; ++f) {
        const int cc = c0 + f;
        if (cc <= cl) {
          const int sl = (unit_begin(cc, P.U, P.C) >= ub) ? 2 * cc : 2 * cc + 1;
          const float* src = P.partials + ((size_t)(sl * NC + warp) * T * 32 + lane) * NACC;
#pragma unroll
          for (int i = 0; i < T; ++i)
#pragma unroll
            for (int e = 0; e < NACC; e += 4)
              q[f][i][e / 4] = ld_relaxed_gpu(reinterpret_cast<const float4*>(src + (size_t)i * 32 * NACC + e));
        }
      }
#pragma unroll
      for (int f = 0; f < kF; ++f) {
        if (c0 + f <= cl) {
#pragma unroll
          for (int i = 0; i < T; ++i)
#pragma unroll
            for (int e = 0; e < NACC; e += 4) {
              s[i][e] += q[f][i][e / 4].x;
              s[i][e + 1] += q[f][i][e / 4].y;
              s[i][e + 2] += q[f][i][e / 4].z;
              s[i][e + 3] += q[f][i][e / 4].w;
            }
        }
      }
    }
    store_y(P, b, warp, lane, tb, s);
    if (lane == 0) P.counters[(size_t)b * NC + warp] = 0u;  // ready for the next call
  }

  // Producer: one lane streams the CTA's units through the ring.  The packed weights and
  // parameters of the first S units are requested before griddepcontrol.wait (they are
  // static, so this may overlap the tail of the kernel before us in the stream); x, which
  // that kernel may have produced, only after it.
  // xmap: the tensor map of x (kernels for M >= 2), in the kernel's parameter space
  __device__ static void produce(const GemvParams& P, const CUtensorMap* xmap, uint8_t* smem,
                                 int u0, int n) {
    const uint32_t ring = smem_addr(smem);
    const uint32_t bars = ring + C_::kBarOff;
    const uint64_t pol = evict_first_policy();
    auto weights = [&](int i, int b, int g) {
      const int s = i % S;
      const int tb = tiles_in_block(b, P.ntiles);
      const long long ch = chunk_index(b, g, 0, P.G, P.ntiles);
      const uint32_t st = ring + s * C_::kStageBytes;
      const uint32_t full = bars + 8 * s;
      const uint32_t code_bytes = tb * C_::kChunkBytes;
      const uint32_t param_bytes = tb * C_::kParamChunk;
      mbar_arrive_expect_tx(full, code_bytes + (kLut || kCb ? 1 : 2) * param_bytes + 256u * P.M);
      bulk_g2s(st, P.qw + ch * C_::kChunkBytes, code_bytes, full, pol);
      if constexpr (kCb) {  // the scales only
        bulk_g2s(st + C_::kCodeBytes, P.sc + ch * 16, param_bytes, full, pol);
      } else if constexpr (kLut) {
        bulk_g2s(st + C_::kCodeBytes, static_cast<const float*>(P.zp) + ch * 32, param_bytes, full,
                 pol);
      } else {
        bulk_g2s(st + C_::kCodeBytes, P.sc + ch * 16 * NS, param_bytes, full, pol);
        bulk_g2s(st + C_::kCodeBytes + C_::kZeroOff, static_cast<const __half*>(P.zp) + ch * 16 * NS,
                 param_bytes, full, pol);
      }
    };
    // the group's M rows of x: one row by a plain bulk copy; M >= 2 rows by one 2-D tensor
    // copy of the box (k = 128 g .. 128 g + 127, every row), 128 g elements being a
    // 256-byte aligned start
    auto activations = [&](int i, int g) {
      const int s = i % S;
      const uint32_t st = ring + s * C_::kStageBytes;
      if constexpr (C_::M1) {
        const __half* xg = P.x + (size_t)g * kGroup;
        for (int m = 0; m < P.M; ++m)
          bulk_g2s(st + C_::kXOff + m * C_::kXStride, xg + (size_t)m * P.K, 256u, bars + 8 * s);
      } else {
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3}], [%4];"
            :: "r"(st + C_::kXOff), "l"(reinterpret_cast<uint64_t>(xmap)), "r"(g * kGroup),
               "r"(0), "r"(bars + 8 * s)
            : "memory");
      }
    };
    if constexpr (TH) {  // tests of the bounded waits: CTA 0's first copy comes late
      if ((P.test_us & 0xFFFFu) && blockIdx.x == 0) test_delay(P.test_us & 0xFFFFu);
    }
    const int b0 = u0 / P.G, g0 = u0 - b0 * P.G;
    int b = b0, g = g0;
    const int pre = n < S ? n : S;
    for (int i = 0; i < pre; ++i) {
      weights(i, b, g);
      if (++g == P.G) {
        g = 0;
        ++b;
      }
    }
    grid_dependency_wait();
    b = b0;
    g = g0;
    for (int i = 0; i < n; ++i) {
      if (i >= S) {
        stage_wait<TH>(P, bars + 8 * (S + i % S), ((i / S) - 1) & 1, kErrEmptyTimeout);
        weights(i, b, g);
      }
      activations(i, g);
      if (++g == P.G) {
        g = 0;
        ++b;
      }
    }
  }

  // One unit (block b, group g) of the CTA's range: warp h of the group takes tiles
  // kTW h .. kTW h + kTW - 1 (of a ragged block, a warp without tiles only releases the
  // stage; tiles past the block's end in a warp's last quad read stale bytes whose sums are
  // never written out).
  __device__ static void unit(const GemvParams& P, uint8_t* smem, int i, int b, int warp,
                              int lane, float (&acc)[kTW][NACC], uint32_t (&orc)[3],
                              uint32_t (&oval)[3], int n) {
    if constexpr (NS > 1) {
      unit_fine(P, smem, i, b, warp, lane, acc);
      return;
    }
    const uint32_t ring = smem_addr(smem);
    const uint32_t bars = ring + C_::kBarOff;
    const uint32_t lut = ring + C_::kLutOff;
    const int sub = warp % WPU;
    const int s = i % S;
    const int tb = tiles_in_block(b, P.ntiles);
    const uint32_t st = ring + s * C_::kStageBytes;
    stage_wait<TH>(P, bars + 8 * s, (i / S) & 1, kErrFullTimeout);
    uint4 xr[4], xr2[4];
    read_x(P, st, lane, xr, xr2);
    if constexpr (OUTL) {
      // outliers of this unit, split over the warps of the group, with x from the stage;
      // then prefetch the group's next unit's
      float* ysm = reinterpret_cast<float*>(smem + C_::kYsmOff);
      const uint32_t* toff = reinterpret_cast<const uint32_t*>(smem + C_::kToffOff);
      const uint32_t e0 = toff[i] + 32 * sub + lane, e1 = toff[i + 1];
      auto add_outlier = [&](uint32_t rc, uint32_t vb) {
        // in-tile position; an out-of-range pair wraps instead of leaving the tile
        const int row = rc & 0x7F, col = (rc >> 8) & 0x7F;
        const float v = __half2float(__ushort_as_half((unsigned short)vb));
        const uint32_t xa = st + C_::kXOff + 2 * row;
        float xv[C_::kXRows];  // all rows' loads in flight before the first atomic
#pragma unroll
        for (int m = 0; m < C_::kXRows; ++m)
          xv[m] = m < P.M ? __half2float(__ushort_as_half(lds16(xa + m * C_::kXStride))) : 0.f;
#pragma unroll
        for (int m = 0; m < C_::kXRows; ++m)
          if (m < P.M) atomicAdd(ysm + m * 128 + col, v * xv[m]);
      };
#pragma unroll
      for (int k = 0; k < kOutPre; ++k)
        if (e0 + 32 * WPU * k < e1) add_outlier(orc[k], oval[k]);
      for (uint32_t e = e0 + 32 * WPU * kOutPre; e < e1; e += 32 * WPU)  // dense tiles
        add_outlier(__ldg(P.tile_rc + e), __ldg(P.tile_val + e));
      prefetch_outliers(P, toff, i + NP, n, 32 * sub + lane, orc, oval);
    }
    const int t0 = kTW * sub;                      // first tile of this warp
    const int nq = tb <= t0 ? 0 : (tb - t0 >= kTW ? kTW / kQ : (tb - t0 + kQ - 1) / kQ);
    const uint32_t empty = bars + 8 * (S + s);
    float cx[NACC];
    auto sum_x = [&]() {
      if constexpr (kLut || kCb) {  // no zero points: no sum of x
#pragma unroll
        for (int e = 0; e < NACC; ++e) cx[e] = 0.f;
      } else {  // sum of x over the group, in the row scales of the codes
        const uint32_t ones[4] = {kOnesLo, Fmt<FMT>::kOnesHi, kOnesLo, Fmt<FMT>::kOnesHi};
        hmma0(&cx[0], ones, xr[0].x, xr[0].y);
        if constexpr (MT == 2) hmma0(&cx[4], ones, xr2[0].x, xr2[0].y);
#pragma unroll
        for (int s8 = 1; s8 < 8; ++s8) {
          const int p = s8 >> 1, h = s8 & 1;
          hmma(&cx[0], ones, h ? xr[p].z : xr[p].x, h ? xr[p].w : xr[p].y);
          if constexpr (MT == 2)
            hmma(&cx[4], ones, h ? xr2[p].z : xr2[p].x, h ? xr2[p].w : xr2[p].y);
        }
      }
    };
    if constexpr (kTW == kQ) {
      // one quad: into registers, release the stage, then the math
      Quad q;
      if (nq) load_quad(st, t0, lane, q);
      __syncwarp();
      if (lane == 0) mbar_arrive(empty);  // this warp's reads of stage s are issued
      if (!nq) return;
      sum_x();
      compute_quad(q, lane, lut, xr, xr2, cx, acc);
    } else {
      // two quads: the stage is released once the last one is in registers, so its refill
      // overlaps that quad's math
      static_assert(kTW == 2 * kQ, "one or two quads per warp");
      sum_x();
      {
        Quad q0;
        load_quad(st, t0, lane, q0);
        if (nq <= 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(empty);
        }
        compute_quad(q0, lane, lut, xr, xr2, cx, acc);
      }
      if (nq > 1) {
        Quad q1;
        load_quad(st, t0 + kQ, lane, q1);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty);
        compute_quad(q1, lane, lut, xr, xr2, cx, acc + kQ);
      }
    }
  }

  // One unit with NS quantization sub-groups (group 64 or 32; W2 / W4 / W8, two warps per
  // unit, two quads of two tiles per warp).  Same stage protocol as unit(); per sub-group:
  // its own sum of x and its own epilogue acc += s (d - z sum x), with that sub-group's
  // scale and zero pairs held in registers (loaded with the codes).
  struct QuadFine {
    uint32_t w[kQ][KW];
    uint32_t p0[kQ][NS], p1[kQ][NS];
  };
  __device__ static void load_quad_fine(uint32_t st, int j0, int lane, QuadFine& r) {
    const int gi = lane >> 2;
#pragma unroll
    for (int i = 0; i < kQ; ++i) {
      const uint32_t cb = st + (j0 + i) * C_::kChunkBytes + lane * 16;
#pragma unroll
      for (int q = 0; q < KW / 4; ++q) {
        const uint4 v = lds128(cb + q * 512);
        r.w[i][4 * q + 0] = v.x;
        r.w[i][4 * q + 1] = v.y;
        r.w[i][4 * q + 2] = v.z;
        r.w[i][4 * q + 3] = v.w;
      }
#pragma unroll
      for (int ss = 0; ss < NS; ++ss) {
        const uint32_t po = ((j0 + i) * NS + ss) * 32 + gi * 4;
        r.p0[i][ss] = lds32(st + C_::kCodeBytes + po);
        r.p1[i][ss] = lds32(st + C_::kCodeBytes + C_::kZeroOff + po);
      }
    }
  }
  __device__ static void compute_quad_fine(const QuadFine& r, const uint4 (&xr)[4],
                                           const uint4 (&xr2)[4], const float (&cx)[NS][NACC],
                                           float (*acc)[NACC]) {
    constexpr int kSub = 8 / NS;  // steps per sub-group
    const auto& w = r.w;
#pragma unroll
    for (int ss = 0; ss < NS; ++ss) {
      float c[kQ][NACC];
      float co[(FMT == kW2) ? kQ : 1][NACC];
#pragma unroll
      for (int s = ss * kSub; s < (ss + 1) * kSub; ++s) {
        const int p = s >> 1, h = s & 1;
        const uint32_t b0 = h ? xr[p].z : xr[p].x, b1 = h ? xr[p].w : xr[p].y;
        uint32_t b2 = 0, b3 = 0;
        if constexpr (MT == 2) {
          b2 = h ? xr2[p].z : xr2[p].x;
          b3 = h ? xr2[p].w : xr2[p].y;
        }
#pragma unroll
        for (int i = 0; i < kQ; ++i) {
          uint32_t a[4];
          frag_uniform<FMT>(w[i], s, a);
          if constexpr (FMT == kW2) {
            if (h == 1) {  // odd steps accumulate separately (their codes carry x16)
              if (s == ss * kSub + 1) {
                hmma0(&co[i][0], a, b0, b1);
                if constexpr (MT == 2) hmma0(&co[i][4], a, b2, b3);
              } else {
                hmma(&co[i][0], a, b0, b1);
                if constexpr (MT == 2) hmma(&co[i][4], a, b2, b3);
              }
              continue;
            }
          }
          if (s == ss * kSub) {
            hmma0(&c[i][0], a, b0, b1);
            if constexpr (MT == 2) hmma0(&c[i][4], a, b2, b3);
          } else {
            hmma(&c[i][0], a, b0, b1);
            if constexpr (MT == 2) hmma(&c[i][4], a, b2, b3);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kQ; ++i) {
        const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&r.p0[i][ss]));
        const float2 z2 = __half22float2(*reinterpret_cast<const __half2*>(&r.p1[i][ss]));
#pragma unroll
        for (int e = 0; e < NACC; ++e) {
          if (C_::M1 && (e & 1)) continue;  // batch column 1 of the fragment: no such row
          float d = c[i][e];
          if constexpr (FMT == kW2) d = fmaf(co[i][e], 0.0625f, d);  // odd steps carry x16
          const float sc = (e & 2) ? s2.y : s2.x;
          const float zc = (e & 2) ? z2.y : z2.x;
          acc[i][e] = fmaf(sc, fmaf(-zc, cx[ss][e], d), acc[i][e]);
        }
      }
    }
  }
  __device__ static void unit_fine(const GemvParams& P, uint8_t* smem, int i, int b, int warp,
                                   int lane, float (&acc)[kTW][NACC]) {
    static_assert(kTW == 2 * kQ, "two quads per warp");
    constexpr int kSub = 8 / NS;
    const uint32_t ring = smem_addr(smem);
    const uint32_t bars = ring + C_::kBarOff;
    const int sub = warp % WPU;
    const int s = i % S;
    const int tb = tiles_in_block(b, P.ntiles);
    const uint32_t st = ring + s * C_::kStageBytes;
    stage_wait<TH>(P, bars + 8 * s, (i / S) & 1, kErrFullTimeout);
    uint4 xr[4], xr2[4];
    read_x(P, st, lane, xr, xr2);
    const int t0 = kTW * sub;
    const int nq = tb <= t0 ? 0 : (tb - t0 >= kTW ? kTW / kQ : (tb - t0 + kQ - 1) / kQ);
    const uint32_t empty = bars + 8 * (S + s);
    // sums of x over each sub-group, in the row scales of the codes
    float cx[NS][NACC];
    {
      const uint32_t ones[4] = {kOnesLo, Fmt<FMT>::kOnesHi, kOnesLo, Fmt<FMT>::kOnesHi};
#pragma unroll
      for (int s8 = 0; s8 < 8; ++s8) {
        const int p = s8 >> 1, h = s8 & 1, ss = s8 / kSub;
        if (s8 % kSub == 0) {
          hmma0(&cx[ss][0], ones, h ? xr[p].z : xr[p].x, h ? xr[p].w : xr[p].y);
          if constexpr (MT == 2)
            hmma0(&cx[ss][4], ones, h ? xr2[p].z : xr2[p].x, h ? xr2[p].w : xr2[p].y);
        } else {
          hmma(&cx[ss][0], ones, h ? xr[p].z : xr[p].x, h ? xr[p].w : xr[p].y);
          if constexpr (MT == 2)
            hmma(&cx[ss][4], ones, h ? xr2[p].z : xr2[p].x, h ? xr2[p].w : xr2[p].y);
        }
      }
    }
    {
      QuadFine q0;
      load_quad_fine(st, t0, lane, q0);
      if (nq <= 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(empty);
      }
      if (nq >= 1) compute_quad_fine(q0, xr, xr2, cx, acc);
    }
    if (nq > 1) {
      QuadFine q1;
      load_quad_fine(st, t0 + kQ, lane, q1);
      __syncwarp();
      if (lane == 0) mbar_arrive(empty);
      compute_quad_fine(q1, xr, xr2, cx, acc + kQ);
    }
  }

  // Entries of unit i a thread takes first (index `slot` of the WPU x 32 threads of the
  // group, then every WPU x 32-th), held in registers one unit ahead.
  static constexpr int kOutPre = 3 - (WPU > 1) - (WPU > 2);
  __device__ static void prefetch_outliers(const GemvParams& P, const uint32_t* toff, int i, int n,
                                           int slot, uint32_t (&orc)[3], uint32_t (&oval)[3]) {
    if (i >= n) return;
#pragma unroll
    for (int k = 0; k < kOutPre; ++k) {
      const uint32_t e = toff[i] + slot + 32 * WPU * k;
      if (e < toff[i + 1]) {
        orc[k] = __ldg(P.tile_rc + e);
        oval[k] = __ldg(P.tile_val + e);
      }
    }
  }

  // Warp group p = warp / WPU takes units i = p, p + NP, ... of the CTA's range (the stages
  // i mod S are then private to it).  At the end of every run of units of one block the
  // warps meet and combine their sums.
  __device__ static void consume(const GemvParams& P, uint8_t* smem, int u0, int n,
                                 int warp, int lane) {
    const int first_block = u0 / P.G;
    const int grp = warp / WPU;
    float acc[kTW][NACC];
#pragma unroll
    for (int j = 0; j < kTW; ++j)
#pragma unroll
      for (int e = 0; e < NACC; ++e) acc[j][e] = 0.f;
    uint32_t orc[3] = {0, 0, 0}, oval[3] = {0, 0, 0};
    // tests of the bounded waits: CTA 0's warp 0 takes stage 0 and holds it for a while
    // before its first unit releases it (waiting for a completed phase again returns at once)
    if constexpr (TH) {
      if ((P.test_us >> 16) && blockIdx.x == 0 && warp == 0 && n > 0) {
        stage_wait<TH>(P, smem_addr(smem) + C_::kBarOff, 0, kErrFullTimeout);
        test_delay(P.test_us >> 16);
      }
    }
    if constexpr (OUTL) {
      consumer_sync(NC * 32);  // the Tile-COO offsets are in shared memory
      prefetch_outliers(P, reinterpret_cast<const uint32_t*>(smem + C_::kToffOff), grp, n,
                        32 * (warp % WPU) + lane, orc, oval);
    }
    int b = first_block, g0 = u0 - first_block * P.G;
    for (int i0 = 0; i0 < n; ++b) {
      const int len = (n - i0) < (P.G - g0) ? (n - i0) : (P.G - g0);
      const int i1 = i0 + len;
      for (int i = i0 + ((grp - i0 % NP) + NP) % NP; i < i1; i += NP)
        unit(P, smem, i, b, warp, lane, acc, orc, oval, n);
      finish_block(P, smem, b, g0 == 0 && len == P.G, first_block, warp, lane, acc);
      i0 = i1;
      g0 = 0;
    }
  }
};

// Second kernel parameter: the tensor map of x for the kernels of M >= 2, an unused word for
// the single-row ones.  (Kept out of GemvParams: a 128-byte grid-constant parameter block
// costs the single-row kernels about 3%.)
struct NoXMap {
  int unused;
};
template <bool XT> struct XMapParam { using type = NoXMap; };
template <> struct XMapParam<true> { using type = CUtensorMap; };

template <int FMT, int MT, bool OUTL, int WPU, bool M1, int OCC, int NS = 1, bool TH = false>
__global__ void __launch_bounds__(Cfg<FMT, MT, OUTL, WPU, M1, OCC, NS>::kThreads,
                                  Cfg<FMT, MT, OUTL, WPU, M1, OCC, NS>::kMinCtas)
    qgemv_kernel(const GemvParams P, const __grid_constant__ typename XMapParam<!M1>::type xm) {
  const CUtensorMap* xmap = nullptr;
  if constexpr (!M1) xmap = &xm;
  using G_ = Gemv<FMT, MT, OUTL, WPU, M1, OCC, NS, TH>;
  using C_ = Cfg<FMT, MT, OUTL, WPU, M1, OCC, NS>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int u0 = unit_begin(blockIdx.x, P.U, P.C);
  const int u1 = unit_begin(blockIdx.x + 1, P.U, P.C);
  const int n = u1 - u0;
  if (threadIdx.x == 0) {
    const uint32_t bars = smem_addr(smem) + C_::kBarOff;
    for (int s = 0; s < C_::S; ++s) {
      mbar_init(bars + 8 * s, 1);            // full: the producer's expect_tx arrival
      mbar_init(bars + 8 * (C_::S + s), C_::WPU);  // empty: the warps of the group
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if constexpr (G_::kLut) {
    build_lut_table(reinterpret_cast<uint32_t*>(smem + C_::kLutOff), P.sc, threadIdx.x,
                    C_::kThreads);
  }
  if constexpr (G_::kCb) {  // the codebook (fp16 [256][4]) arrives in P.zp
    build_cb_table(reinterpret_cast<uint2*>(smem + C_::kLutOff), static_cast<const __half*>(P.zp),
                   threadIdx.x, C_::kThreads);
  }
  // x rows M .. kXRows-1 of every stage are never copied: keep them zero (16-byte stores,
  // rows are 256 bytes)
  {
    const int chunks = (C_::kXRows - (P.M < C_::kXRows ? P.M : C_::kXRows)) * (C_::kXStride / 16);
#pragma unroll
    for (int st = 0; st < C_::S; ++st) {
      uint4* z = reinterpret_cast<uint4*>(smem + st * C_::kStageBytes + C_::kXOff + P.M * C_::kXStride);
      for (int e = threadIdx.x; e < chunks; e += C_::kThreads) z[e] = make_uint4(0, 0, 0, 0);
    }
  }
  if constexpr (OUTL) {
    float* ysm = reinterpret_cast<float*>(smem + C_::kYsmOff);
    for (int i = threadIdx.x; i < 16 * 128; i += C_::kThreads) ysm[i] = 0.f;
  }
  __syncthreads();
  grid_dependents_launch();
  if (warp == C_::NC) {
    if (lane == 0) G_::produce(P, xmap, smem, u0, n);
    return;
  }
  if constexpr (OUTL) {
    // the range's Tile-COO offsets (static data, like the weights), fetched while the
    // first stages fill; consume() meets on a barrier before reading them
    uint32_t* toff = reinterpret_cast<uint32_t*>(smem + C_::kToffOff);
    for (int i = threadIdx.x; i <= n; i += C_::NC * 32) toff[i] = __ldg(P.tile_off + u0 + i);
  }
  grid_dependency_wait();  // x, y and the workspace may belong to the kernel before us
  G_::consume(P, smem, u0, n, warp, lane);
}


}  // namespace qlk
