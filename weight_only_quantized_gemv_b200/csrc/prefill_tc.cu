// Prefill GEMM on the fifth-generation tensor cores (tcgen05), sm_100a:
//
//   y[M][N] = x[M][K] . W[N][K]^T,   fp16 operands, fp32 accumulation in tensor memory,
//                                    fp16 round-to-nearest-even output
//
// For M >> 16 the layer is compute-bound (QFactory page, assumption stress test and
// limitation 1), and the weights are dequantized once per tile instead of once per 16 rows
// of x.  Two forms of the A operand (the weights):
//  * FUSED: producer warps read the packed codes and their scales / zeros (absmax) from
//    global memory, dequantize them in registers to the same fp16 values the stand-alone
//    dequantization writes ("Fast NF4 Dequantization Kernels" page, method section: codes
//    -> FP16 -> matmul; here FP16 goes to shared memory instead of back to HBM), and store
//    them into the shared-memory operand of the MMAs;
//  * dense: a TMA tensor copy of an fp16 W[N][K] (the stand-alone dequantization's output).
//
// Design:
//  * One persistent CTA per SM; output tiles of 128 weight rows (the MMA's M: output
//    columns n) x BN rows of x (the MMA's N: tokens), taken in turn by the CTAs.
//  * A ring of S shared-memory stages of 64 k each: A 128 x 64 and B BN x 64 fp16, both in
//    the K-major 128-byte-swizzled layout (rows of 128 bytes, 16-byte granule c of row r at
//    granule c ^ (r mod 8)), which is what the TMA copy with 128-byte swizzle writes.
//  * Warp 0: one lane issues the TMA copies (x, and W in the dense form).  Warp 1: one lane
//    issues tcgen05.mma (M = 128, N = BN, K = 16; four per stage) and tcgen05.commit, which
//    releases a stage once the MMAs that read it are done; the warp owns the tensor memory.
//    Warps 2..5: epilogue (tcgen05.ld of the accumulator, fp16 stores).  FUSED: warps
//    6..13 dequantize (one 16-column tile of the 128 rows each).
//  * Two accumulators of BN fp32 columns in tensor memory: the epilogue of one tile
//    overlaps the MMAs of the next.
//  * Every mbarrier wait is bounded in time (100 ms; a healthy one takes microseconds).  One
//    that runs out sets a flag in a device error word (qlinear_prefill_read_error) and a
//    CTA-wide abort flag; every role then leaves its loop, waits briefly for its copies and
//    MMAs in flight, and the CTA releases its tensor memory and exits.  A lost copy gives
//    wrong numbers, never a hung GPU.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <unordered_map>

#include "dequant_frag.cuh"
#include "kernels.cuh"
#include "layout.h"
#include "qlinear.h"

using namespace qlayout;

namespace {

constexpr int kBM = 128;  // weight rows per tile (MMA M)
constexpr int kBK = 64;   // k per stage: one 128-byte swizzle atom of fp16
constexpr int kDqWarps = 8;
constexpr uint32_t kErrStage = 1u, kErrAcc = 2u;

__device__ uint32_t g_tc_err;  // sticky wait-timeout flags of the prefill kernels

template <int BN, bool FUSED, int FMT = kW4>
struct TcCfg {
  static_assert(BN == 128 || BN == 256, "token tile");
  static constexpr int kABytes = kBM * kBK * 2;              // 16 KB
  static constexpr int kBBytes = BN * kBK * 2;               // 32 / 16 KB
  // FUSED: the stage's packed codes, as bulk-copied: per 16-row tile the half chunk of the
  // stage's 64 k (W4, LUT4: quad h, 512 B; W8: quads 2h, 2h + 1, 1 KB; W2: the whole 512-B
  // chunk, whose halves interleave per lane), then the block's parameters for the group
  // (scales and zeros 8 x 32 B each; LUT4: absmax 8 x 128 B)
  static constexpr int kCodeChunk = FMT == kW8 ? 1024 : 512;
  static constexpr int kCodeBytes = FUSED ? 8 * kCodeChunk : 0;
  static constexpr int kParChunk = FMT == kLUT4 ? 128 : 32;  // per tile, per array
  static constexpr int kParBytes = FUSED ? (FMT == kLUT4 ? 8 * 128 : 2 * 8 * 32) : 0;
  static constexpr int kCodeOff = kABytes + kBBytes;
  static constexpr int kParOff = kCodeOff + kCodeBytes;
  static constexpr int kStageBytes = (kParOff + kParBytes + 1023) / 1024 * 1024;
  static constexpr int S0 = (232448 - 2048) / kStageBytes;   // stages that fit
  static constexpr int S = S0 < 6 ? S0 : 6;
  static_assert(S >= 3, "pipeline depth");
  static constexpr int kEpiWarp0 = 2, kEpiWarps = 4;
  static constexpr int kDqWarp0 = kEpiWarp0 + kEpiWarps;
  static constexpr int kWarps = kDqWarp0 + (FUSED ? kDqWarps : 0);
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kBarOff = S * kStageBytes;
  // full[S] empty[S] accf[2] acce[2] fin cfull[S]
  static constexpr int kSlotOff = kBarOff + 8 * (3 * S + 5);  // tensor-memory base, abort flag
  static constexpr int kSmemBytes = kSlotOff + 16 + 1024;    // + slack to align the ring
  static constexpr uint32_t kTmemCols = 2 * BN;
  // full[s] completes on the TMA bytes of x (and W) plus one arrival per dequantizing warp;
  // cfull[s] (FUSED) on the bytes of the stage's codes and parameters
  static constexpr uint32_t kFullCount = 1 + (FUSED ? kDqWarps : 0);
};

struct TcParams {
  const uint8_t* qw;     // FUSED: packed codes
  const void* p0;        // FUSED: packed scales | lut16
  const void* p1;        // FUSED: packed zeros | packed absmax
  __half* y;             // [M][N]
  float* partials;       // stream-K: fp32 partial tiles, two slots per CTA (null: whole tiles)
  uint32_t* counters;    // stream-K: arrivals per (tile, epilogue warp)
  int M, N, K, G, ntiles, mtiles, tiles;
};

// The k-block work of a CTA as a sequence of segments (tile t, k-blocks [kb0, kb1)).
//  * whole tiles (no partials): tiles c, c + C, c + 2C, ... each from k-block 0 to KB;
//  * stream-K: the flattened (tile, k-block) units [c U / C, (c + 1) U / C), U = tiles x KB,
//    cut at tile boundaries: only a CTA's first and last segments can be partial tiles,
//    and every CTA gets the same number of k-blocks to within one.
struct SegIter {
  long long u, u1;  // stream-K: next unit, end of the range
  int j;            // whole tiles: next tile of this CTA
  __device__ void init(const TcParams& P, int KB) {
    const long long U = (long long)P.tiles * KB, C = gridDim.x;
    u = blockIdx.x * U / C;
    u1 = (blockIdx.x + 1) * U / C;
    j = 0;
  }
  __device__ bool next(const TcParams& P, int KB, int& t, int& kb0, int& kb1) {
    if (P.partials) {
      if (u >= u1) return false;
      t = (int)(u / KB);
      kb0 = (int)(u - (long long)t * KB);
      kb1 = (u1 - u < (long long)(KB - kb0)) ? kb0 + (int)(u1 - u) : KB;
      u += kb1 - kb0;
      return true;
    }
    t = blockIdx.x + j * gridDim.x;
    if (t >= P.tiles) return false;
    ++j;
    kb0 = 0;
    kb1 = KB;
    return true;
  }
};

// stream-K: the CTA whose unit range holds unit u
__device__ __forceinline__ int sk_cta_of(long long u, long long U, int C) {
  return (int)(((u + 1) * C - 1) / U);
}
__device__ __forceinline__ long long sk_begin(int c, long long U, int C) { return c * U / C; }

// ---------------------------------------------------------------------------
// tcgen05 / TMA helpers

__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// D[tmem] (+)= A[smem] . B[smem]^T, both K-major (shape in the instruction descriptor)
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}
// Instruction descriptor of kind::f16: fp16 A and B (K-major), fp32 D, M x N.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                       uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ldg_nc128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ldg_nc64(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_nc32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with parity `parity` of `bar`.  A healthy wait here lasts microseconds;
// this one gives up after `limit_ns`, or as soon as another role of the CTA has given up
// (*abort set; the waits of the teardown ignore it), and then sets `bit` in the error word
// and *abort, and returns false.  Every
// role leaves its loop on the first failed wait, so a broken pipeline ends the kernel within
// a few limits instead of one limit per remaining wait.
constexpr uint64_t kWaitNs = 100ull * 1000 * 1000;
__device__ __noinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                     uint32_t bit, uint64_t limit_ns = kWaitNs,
                                     bool honor_abort = true, bool patient = false,
                                     uint32_t backoff_ns = 0) {
  // The first kSpin rounds poll, sleeping backoff_ns between polls (the pipeline's waits are
  // usually short; the sleep keeps a polling lane from taking the issue slots of the warps
  // that do the work); after that each try_wait may suspend the thread for up to kSuspendNs
  // until the phase completes.  `patient` waiters (the epilogue, whose waits last a whole
  // tile) suspend from the start.
  constexpr uint32_t kSpin = 2048, kSuspendNs = 500;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = patient ? kSpin : 0;; ++it) {
    uint32_t done;
    if (it < kSpin) {
      asm volatile(
          "{\n\t.reg .pred p;\n\t"
          "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(done)
          : "r"(bar), "r"(parity)
          : "memory");
    } else {
      asm volatile(
          "{\n\t.reg .pred p;\n\t"
          "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(done)
          : "r"(bar), "r"(parity), "r"(kSuspendNs)
          : "memory");
    }
    if (done) return true;
    // past the first polls, sleep between them: leave the issue slots to the working warps
    if (backoff_ns && it >= 256 && it < kSpin) __nanosleep(backoff_ns);
    if ((it & 63u) == 63u) {
      if ((honor_abort && *abort) || globaltimer_ns() - t0 > limit_ns) break;
    }
  }
  atomicOr(&g_tc_err, bit);
  *abort = 1u;
  return false;
}

// ---------------------------------------------------------------------------
// FUSED: one dequantizing warp's share of a stage: tile jj (16 weight rows) of the 128-row
// block, k = 64 kb .. 64 kb + 63 (half kb % 2 of group kb / 2).

template <int FMT>
struct DqFrag {
  static constexpr int KWL = FMT == kW2 ? 2 : FMT == kW8 ? 8 : 4;  // words of four steps
  uint32_t w[KWL];
  uint32_t p0, p1;  // scale and zero pairs (uniform) | absmax of rows gi, gi + 8 (LUT4)
};

// The stage's codes and parameters of tile jj, from shared memory (bulk-copied by the TMA
// lane; layouts as in TcCfg): `st` = the stage, `half` = kb % 2.
template <int FMT, class C>
__device__ __forceinline__ void dq_load_smem(uint32_t st, int jj, int half, int lane,
                                             DqFrag<FMT>& f) {
  const int gi = lane >> 2;
  const uint32_t c = st + C::kCodeOff + jj * C::kCodeChunk;
  if constexpr (FMT == kW2) {  // the whole chunk: steps 4 half .. 4 half + 3 = words 2 half, +1
    const uint2 v = qlk::lds64(c + lane * 16 + half * 8);
    f.w[0] = v.x;
    f.w[1] = v.y;
  } else if constexpr (FMT == kW8) {  // quads 2 half, 2 half + 1
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 v = qlk::lds128(c + (q * 32 + lane) * 16);
      f.w[4 * q] = v.x;
      f.w[4 * q + 1] = v.y;
      f.w[4 * q + 2] = v.z;
      f.w[4 * q + 3] = v.w;
    }
  } else {  // W4, LUT4: quad `half`
    const uint4 v = qlk::lds128(c + lane * 16);
    f.w[0] = v.x;
    f.w[1] = v.y;
    f.w[2] = v.z;
    f.w[3] = v.w;
  }
  const uint32_t pa = st + C::kParOff;
  if constexpr (FMT == kLUT4) {  // absmax of (rows gi, gi + 8) for this half's 64-block
    const uint2 v = qlk::lds64(pa + jj * 128 + gi * 16 + half * 8);
    f.p0 = v.x;
    f.p1 = v.y;
  } else {
    f.p0 = qlk::lds32(pa + jj * 32 + gi * 4);
    f.p1 = qlk::lds32(pa + 8 * 32 + jj * 32 + gi * 4);
  }
}

// Decode and store into the stage's A operand: row 16 jj + gi + 8 h, k granule 4 i + t.
// The eight lanes of a store phase (gi = 2p, 2p + 1; t = 0..3) write rows gi of one granule
// half each; lanes with odd gi exchange their two step pairs (the words of steps 0, 1 and
// of steps 2, 3: same step parities, so the same decode) and store the halves in the
// opposite order, so that the eight 16-byte granules of a phase are distinct (c ^ gi covers
// both halves): conflict-free.  The exchange is on the words, before the decode, and
// branch-free.
template <int FMT>
__device__ __forceinline__ void dq_store(const DqFrag<FMT>& f, uint32_t a_base, int jj, int lane,
                                         const float* lut_s) {
  const int gi = lane >> 2, t = lane & 3;
  const uint32_t swap = (uint32_t)(gi & 1), m = 0u - swap;
  constexpr int HW = DqFrag<FMT>::KWL / 2;
  uint32_t w[DqFrag<FMT>::KWL];
#pragma unroll
  for (int k = 0; k < HW; ++k) {
    w[k] = (f.w[k + HW] & m) | (f.w[k] & ~m);
    w[k + HW] = (f.w[k] & m) | (f.w[k + HW] & ~m);
  }
  __half2 zb[2][2];
  __half2 s_lo, s_hi;
  if constexpr (FMT != kLUT4) {
    const __half2 s2 = qdq::u32_as_h2(f.p0), z2 = qdq::u32_as_h2(f.p1);
    qdq::zero_bias<FMT>(__low2float(z2), __high2float(z2), zb);
    s_lo = __low2half2(s2);
    s_hi = __high2half2(s2);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4 val;
      if constexpr (FMT == kLUT4)
        val = qdq::lut_pair8(w, 2 * i, h, lut_s, __uint_as_float(h ? f.p1 : f.p0));
      else
        val = qdq::uniform_pair8<FMT>(w, 2 * i, h, zb, h ? s_hi : s_lo);
      const int row = 16 * jj + gi + 8 * h;
      sts128(a_base + row * 128 + (((4 * (i ^ (int)swap) + t) ^ gi) << 4), val);
    }
}

// ---------------------------------------------------------------------------

// FUSED: tensor maps over the packed codes and parameters as 2-D arrays [chunk][words]:
// one copy brings the stage's rows of the block's 8 chunks (a box of 8 chunk rows).
struct CodeMaps {
  CUtensorMap codes, p0, p1;
};

template <int BN, bool FUSED, int FMT>
__global__ void __launch_bounds__(TcCfg<BN, FUSED, FMT>::kThreads, 1)
    prefill_tc_kernel(const TcParams P, const __grid_constant__ CUtensorMap xmap,
                      const __grid_constant__ CUtensorMap wmap,
                      const __grid_constant__ CodeMaps cmaps) {
  using C = TcCfg<BN, FUSED, FMT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = qlk::smem_addr(smem_raw);
  const uint32_t ring = (raw + 1023u) & ~1023u;  // the swizzled layout wants 1024-byte atoms
  uint8_t* smem = smem_raw + (ring - raw);
  const uint32_t bars = ring + C::kBarOff;
  auto full = [&](int s) { return bars + 8 * s; };
  auto empty = [&](int s) { return bars + 8 * (C::S + s); };
  auto accf = [&](int a) { return bars + 8 * (2 * C::S + a); };
  auto acce = [&](int a) { return bars + 8 * (2 * C::S + 2 + a); };
  const uint32_t fin = bars + 8 * (2 * C::S + 4);  // the last MMAs' completion
  auto cfull = [&](int s) { return bars + 8 * (2 * C::S + 5 + s); };  // FUSED: codes landed
  const uint32_t slot = ring + C::kSlotOff;
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + C::kSlotOff + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = P.K / kBK;

  __shared__ float lut_s[16];
  if (FUSED && FMT == kLUT4 && threadIdx.x < 16)
    lut_s[threadIdx.x] = __half2float(static_cast<const __half*>(P.p0)[threadIdx.x]);
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::S; ++s) {
      qlk::mbar_init(full(s), C::kFullCount);
      qlk::mbar_init(empty(s), 1);
      qlk::mbar_init(cfull(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      qlk::mbar_init(accf(a), 1);
      qlk::mbar_init(acce(a), C::kEpiWarps);
    }
    qlk::mbar_init(fin, 1);
    *abort = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::kSlotOff);

  if (warp == 0) {
    // ---- TMA producer
    if (lane == 0) {
      int it = 0, t, kb0, kb1;
      bool ok = true;
      SegIter sg;
      sg.init(P, KB);
      while (ok && sg.next(P, KB, t, kb0, kb1)) {
        const int nt = t / P.mtiles, mt = t - nt * P.mtiles;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % C::S;
          if (it >= C::S &&
              !(ok = tc_wait(empty(s), ((it / C::S) - 1) & 1, abort, kErrStage, kWaitNs, true,
                             false, 64)))
            break;
          const uint32_t st = ring + s * C::kStageBytes;
          if constexpr (FUSED) {
            // the stage's packed codes (rows: the block's 8 chunks of the group, columns: the
            // stage's half, or all of a W2 chunk) and the group's parameters, three tensor
            // copies; rows past the block are another group's (unused) or read as zeros
            const int g = kb >> 1, half = kb & 1;
            const int ch0 = (int)chunk_index(nt, g, 0, P.G, P.ntiles);
            qlk::mbar_arrive_expect_tx(cfull(s), C::kCodeBytes + C::kParBytes);
            tma_2d(st + C::kCodeOff, &cmaps.codes, FMT == kW2 ? 0 : half * (C::kCodeChunk / 4), ch0,
                   cfull(s));
            if constexpr (FMT == kLUT4) {
              tma_2d(st + C::kParOff, &cmaps.p1, 0, ch0, cfull(s));
            } else {
              tma_2d(st + C::kParOff, &cmaps.p0, 0, ch0, cfull(s));
              tma_2d(st + C::kParOff + 8 * 32, &cmaps.p1, 0, ch0, cfull(s));
            }
          }
          qlk::mbar_arrive_expect_tx(full(s), C::kBBytes + (FUSED ? 0 : C::kABytes));
          tma_2d(st + C::kABytes, &xmap, kb * kBK, mt * BN, full(s));
          if constexpr (!FUSED) tma_2d(st, &wmap, kb * kBK, nt * kBM, full(s));
        }
      }
      // no copy of this CTA is still in flight when it exits: wait for the last stages filled
      for (int i = (it > C::S ? it - C::S : 0); i < it; ++i) {
        tc_wait(full(i % C::S), (i / C::S) & 1, abort, kErrStage, kWaitNs / 10, false);
        if (FUSED) tc_wait(cfull(i % C::S), (i / C::S) & 1, abort, kErrStage, kWaitNs / 10, false);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(kBM, BN);
      int it = 0, j = 0, t, kb0, kb1;
      bool ok = true;
      SegIter sg;
      sg.init(P, KB);
      for (; ok && sg.next(P, KB, t, kb0, kb1); ++j) {
        const int a = j & 1;
        if (j >= 2 && !(ok = tc_wait(acce(a), ((j >> 1) - 1) & 1, abort, kErrAcc))) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * BN);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % C::S;
          if (!(ok = tc_wait(full(s), (it / C::S) & 1, abort, kErrStage, kWaitNs, true, false, 32)))
            break;
          tc_fence_after();
          const uint32_t st = ring + s * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma(d, desc_sw128(st + 32 * kk), desc_sw128(st + C::kABytes + 32 * kk), idesc,
                   (kb != kb0) || (kk != 0));
          tc_commit(empty(s));  // the stage is free once these MMAs have read it
        }
        if (ok) tc_commit(accf(a));  // the segment's accumulator is complete
      }
      // every MMA issued has completed before the tensor memory is released
      tc_commit(fin);
      tc_wait(fin, 0, abort, kErrAcc, kWaitNs / 10, false);
    }
  } else if (warp < C::kDqWarp0) {
    // ---- epilogue: warp w reads accumulator lanes 32 (w % 4) .. + 31 (weight rows)
    const int q = warp & 3;
    const long long U = (long long)P.tiles * KB;
    const int Cg = gridDim.x;
    int j = 0, t, kb0, kb1;
    SegIter sg;
    sg.init(P, KB);
    for (; sg.next(P, KB, t, kb0, kb1); ++j) {
      const int a = j & 1;
      const int nt = t / P.mtiles, mt = t - nt * P.mtiles;
      bool ok = true;
      if (lane == 0) ok = tc_wait(accf(a), (j >> 1) & 1, abort, kErrAcc, kWaitNs, true, true);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after();
      const int row = 32 * q + lane;
      const int n = nt * kBM + row;
      const int m0 = mt * BN;
      const int cols = (P.M - m0) < BN ? (P.M - m0) : BN;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * BN);
      if (kb0 == 0 && kb1 == KB) {  // the whole tile: round and store
        for (int c0 = 0; c0 < cols; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(tbase + (uint32_t)c0, r);
          tc_wait_ld();
          if (n < P.N) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (c0 + e < cols) P.y[(size_t)(m0 + c0 + e) * P.N + n] = __float2half_rn(__uint_as_float(r[e]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) qlk::mbar_arrive(acce(a));
        continue;
      }
      // part of a tile (stream-K): publish this CTA's fp32 partial; the last contributor
      // adds all of them in CTA order and stores y (nobody waits for anybody)
      const int slot = 2 * (int)blockIdx.x + (j == 0 ? 0 : 1);
      float* mine = P.partials + ((size_t)slot * kBM + row) * BN;
      for (int c0 = 0; c0 < cols; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(tbase + (uint32_t)c0, r);
        tc_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<uint4*>(mine + c0 + e) = make_uint4(r[e], r[e + 1], r[e + 2], r[e + 3]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) qlk::mbar_arrive(acce(a));  // the accumulator is free again
      const int cf = sk_cta_of((long long)t * KB, U, Cg);
      const int cl = sk_cta_of((long long)(t + 1) * KB - 1, U, Cg);
      uint32_t prev = 0;
      if (lane == 0) prev = qlk::arrive_acq_rel(P.counters + (size_t)t * 4 + q);
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev + 1 != (uint32_t)(cl - cf + 1)) continue;
      __syncwarp();
      for (int c0 = 0; c0 < cols; c0 += 16) {
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
        for (int cc = cf; cc <= cl; ++cc) {
          const int sl = (sk_begin(cc, U, Cg) >= (long long)t * KB) ? 2 * cc : 2 * cc + 1;
          const float* src = P.partials + ((size_t)sl * kBM + row) * BN + c0;
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            const float4 v = qlk::ld_relaxed_gpu(reinterpret_cast<const float4*>(src + e));
            acc[e] += v.x;
            acc[e + 1] += v.y;
            acc[e + 2] += v.z;
            acc[e + 3] += v.w;
          }
        }
        if (n < P.N) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (c0 + e < cols) P.y[(size_t)(m0 + c0 + e) * P.N + n] = __float2half_rn(acc[e]);
        }
      }
      if (lane == 0) P.counters[(size_t)t * 4 + q] = 0u;  // ready for the next call
    }
  } else if constexpr (FUSED) {
    // ---- dequantizing producers: warp dw fills rows 16 dw .. 16 dw + 15 of A from the
    // codes the TMA lane brought into the same stage
    const int dw = warp - C::kDqWarp0;
    int it = 0, t, kb0, kb1;
    bool ok = true;
    SegIter sg;
    sg.init(P, KB);
    while (ok && sg.next(P, KB, t, kb0, kb1)) {
      const int tb = tiles_in_block(t / P.mtiles, P.ntiles);
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const int s = it % C::S;
        if (lane == 0)
          ok = tc_wait(cfull(s), (it / C::S) & 1, abort, kErrStage, kWaitNs, true, false, 32);
        if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
        const uint32_t st = ring + s * C::kStageBytes;
        if (dw < tb) {
          DqFrag<FMT> f;
          dq_load_smem<FMT, C>(st, dw, kb & 1, lane, f);
          dq_store<FMT>(f, st, dw, lane, lut_s);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the MMAs
        __syncwarp();
        if (lane == 0) qlk::mbar_arrive(full(s));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// fp16 [rows][K] row-major as a 2-D tensor (K innermost), box 64 k x box_rows, 128-byte
// swizzle.  Rows past the end read as zeros.
bool encode_kmajor(CUtensorMap* map, const void* base, int rows, int K, int box_rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A 2-D array of `rows` rows of `cols` 32-bit words (row stride cols words), box 8 rows x
// box_cols words, no swizzle; rows past the end read as zeros.
bool encode_rows(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int cols,
                 long long rows, int box_cols) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, 8};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, bool FUSED, int FMT>
ql_status launch_tc(const TcParams& P, const void* x, const void* w, cudaStream_t st) {
  using C = TcCfg<BN, FUSED, FMT>;
  auto fn = prefill_tc_kernel<BN, FUSED, FMT>;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QL_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return QL_ERR_CUDA;
  {
    static std::mutex mu;
    static std::unordered_map<int, bool> ready;
    std::lock_guard<std::mutex> lk(mu);
    if (!ready[dev]) {
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
          cudaSuccess)
        return QL_ERR_CUDA;
      int occ = 0;  // the CTA (threads x registers, shared memory) must fit on an SM
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, C::kThreads, C::kSmemBytes) !=
              cudaSuccess ||
          occ < 1)
        return QL_ERR_CUDA;
      ready[dev] = true;
    }
  }
  CUtensorMap xmap, wmap;
  CodeMaps cm;
  if (!encode_kmajor(&xmap, x, P.M, P.K, BN)) return QL_ERR_CUDA;
  if (FUSED) {
    wmap = xmap;  // unused
    const long long nchunks = (long long)P.ntiles * P.G;
    if (!encode_rows(&cm.codes, P.qw, CU_TENSOR_MAP_DATA_TYPE_UINT32, chunk_bytes(FMT) / 4,
                     nchunks, C::kCodeChunk / 4))
      return QL_ERR_CUDA;
    if (FMT == kLUT4) {  // absmax, 32 floats per chunk; p0 (the table) is read directly
      if (!encode_rows(&cm.p1, P.p1, CU_TENSOR_MAP_DATA_TYPE_UINT32, 32, nchunks, 32))
        return QL_ERR_CUDA;
      cm.p0 = cm.p1;
    } else {  // scales, zeros: 16 halves (8 words) per chunk
      if (!encode_rows(&cm.p0, P.p0, CU_TENSOR_MAP_DATA_TYPE_UINT32, 8, nchunks, 8) ||
          !encode_rows(&cm.p1, P.p1, CU_TENSOR_MAP_DATA_TYPE_UINT32, 8, nchunks, 8))
        return QL_ERR_CUDA;
    }
  } else if (!encode_kmajor(&wmap, w, P.N, P.K, kBM)) {
    return QL_ERR_CUDA;
  } else {
    cm.codes = cm.p0 = cm.p1 = xmap;  // unused
  }
  // stream-K: one CTA per SM (at most one per k-block, so that every CTA has work: the
  // fix-up counts the CTAs whose ranges meet a tile), the k-blocks shared out evenly; whole
  // tiles: at most one CTA per tile
  const long long units = P.partials ? (long long)P.tiles * (P.K / kBK) : P.tiles;
  const int grid = units < sms ? (int)units : sms;
  fn<<<grid, C::kThreads, C::kSmemBytes, st>>>(P, xmap, wmap, cm);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

template <bool FUSED, int FMT>
ql_status launch_bn(const TcParams& P, const void* x, const void* w, cudaStream_t st) {
  return P.M <= 128 ? launch_tc<128, FUSED, FMT>(P, x, w, st) : launch_tc<256, FUSED, FMT>(P, x, w, st);
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

TcParams make_params(const void* packed, const void* p0, const void* p1, void* y, int M, int N,
                     int K) {
  TcParams P;
  P.qw = static_cast<const uint8_t*>(packed);
  P.p0 = p0;
  P.p1 = p1;
  P.y = static_cast<__half*>(y);
  P.M = M;
  P.N = N;
  P.K = K;
  P.G = K / kGroup;
  P.ntiles = N / kTileN;
  const int bn = M <= 128 ? 128 : 256;
  P.mtiles = (M + bn - 1) / bn;
  P.tiles = ((N + kBM - 1) / kBM) * P.mtiles;
  P.partials = nullptr;
  P.counters = nullptr;
  return P;
}

// Workspace of the stream-K schedule: arrival counters (one per tile and epilogue warp, zero
// between calls) and two fp32 partial tiles (128 x BN) per CTA.
struct SkLayout {
  size_t counter_bytes, partial_offset, bytes;
};
SkLayout sk_layout(int M, int N, int sms) {
  const int bn = M <= 128 ? 128 : 256;
  const long long tiles = (long long)((N + kBM - 1) / kBM) * ((M + bn - 1) / bn);
  SkLayout L;
  L.counter_bytes = (size_t)tiles * 4 * sizeof(uint32_t);
  L.partial_offset = (L.counter_bytes + 255) / 256 * 256;
  L.bytes = L.partial_offset + (size_t)2 * sms * kBM * bn * sizeof(float);
  return L;
}

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

}  // namespace

// Dense fp16 GEMM on the tensor cores: y[M][N] = x[M][K] . w[N][K]^T (used by
// qlinear_prefill after the stand-alone dequantization).
ql_status qlinear_gemm_f16_tc(const uint16_t* x, const uint16_t* w, uint16_t* y, int M, int N,
                              int K, cudaStream_t st) {
  if (!x || !w || !y) return QL_ERR_NULL;
  if (M < 1 || N < kTileN || N % kTileN || K < kGroup || K % kGroup) return QL_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 2)) return QL_ERR_ALIGN;
  const TcParams P = make_params(nullptr, nullptr, nullptr, y, M, N, K);
  return launch_bn<false, kW4>(P, x, w, st);
}

extern "C" size_t qlinear_prefill_workspace_bytes(int M, int N, int K) {
  if (M < 1 || N < kTileN || N % kTileN || K < kGroup || K % kGroup) return 0;
  const int sms = sm_count();
  return sms > 0 ? sk_layout(M, N, sms).bytes : 0;
}

extern "C" ql_status qlinear_prefill_fused(int fmt, const uint16_t* x, const void* packed,
                                           const void* p0, const void* p1, uint16_t* y, int M,
                                           int N, int K, void* workspace, size_t workspace_bytes,
                                           ql_stream_t stream) {
  if (fmt != kW2 && fmt != kW4 && fmt != kW8 && fmt != kLUT4) return QL_ERR_UNSUPPORTED;
  if (!x || !packed || !p0 || !p1 || !y) return QL_ERR_NULL;
  if (M < 1 || N < kTileN || N % kTileN || K < kGroup || K % kGroup) return QL_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(y, 2)) return QL_ERR_ALIGN;
  // codes and parameters arrive by tensor copies (16-byte aligned bases); the LUT is read
  // directly
  if (fmt == kLUT4 ? (!aligned(p0, 2) || !aligned(p1, 16)) : (!aligned(p0, 16) || !aligned(p1, 16)))
    return QL_ERR_ALIGN;
  TcParams P = make_params(packed, p0, p1, y, M, N, K);
  if (workspace) {  // stream-K
    const int sms = sm_count();
    if (sms <= 0) return QL_ERR_CUDA;
    const SkLayout L = sk_layout(M, N, sms);
    if (workspace_bytes < L.bytes) return QL_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return QL_ERR_ALIGN;
    P.counters = static_cast<uint32_t*>(workspace);
    P.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + L.partial_offset);
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (fmt) {
    case kW2: return launch_bn<true, kW2>(P, x, nullptr, st);
    case kW4: return launch_bn<true, kW4>(P, x, nullptr, st);
    case kW8: return launch_bn<true, kW8>(P, x, nullptr, st);
    default: return launch_bn<true, kLUT4>(P, x, nullptr, st);
  }
}

extern "C" ql_status qlinear_prefill_read_error(uint32_t* flags, ql_stream_t stream) {
  if (!flags) return QL_ERR_NULL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyFromSymbolAsync(flags, g_tc_err, sizeof(uint32_t), 0, cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return QL_ERR_CUDA;
  static const uint32_t zero = 0;
  if (cudaMemcpyToSymbolAsync(g_tc_err, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return QL_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}
