// Prefill GEMM on the fifth-generation tensor cores (tcgen05), sm_100a:
//
//   y[M][N] = x[M][K] . W[N][K]^T,   fp16 operands, fp32 accumulation in tensor memory,
//                                    fp16 round-to-nearest-even output
//
// For M >> 16 the layer is compute-bound (QFactory page, assumption stress test and
// limitation 1), and the weights are dequantized once per tile instead of once per 16 rows
// of x.  Two forms of the A operand (the weights):
//  * FUSED: dequantizing warps decode the packed codes and their scales / zeros (absmax),
//    which a producer warp brings into shared memory by TMA, to the same fp16 values the
//    stand-alone dequantization writes ("Fast NF4 Dequantization Kernels" page, method
//    section: codes -> FP16 -> matmul; here FP16 goes to shared memory instead of back to
//    HBM), and store them into the shared-memory operand of the MMAs;
//  * dense: a TMA tensor copy of an fp16 W[N][K] (the stand-alone dequantization's output).
//
// Design:
//  * One persistent CTA per SM (or cluster pair of CTAs on two SMs: tcgen05 cta_group::2,
//    256-row tiles); output tiles of 128 weight rows per CTA (the MMA's M: output columns n)
//    x BN rows of x (the MMA's N: tokens), taken in turn by the CTAs, or shared out by
//    k-block with a workspace (stream-K).
//  * A ring of S shared-memory stages of 64 k each: A 128 x 64 and B (BN / CTAs) x 64 fp16,
//    both in the K-major 128-byte-swizzled layout (rows of 128 bytes, 16-byte granule c of
//    row r at granule c ^ (r mod 8)), which is what the TMA copy with 128-byte swizzle
//    writes.  FUSED: the codes in a ring of their own, filled ahead of the stages.
//  * Warp 0: one lane issues the TMA copies (x, and W in the dense form).  Warp 1: one lane
//    issues tcgen05.mma (K = 16; four per stage) and tcgen05.commit, which releases a stage
//    once the MMAs that read it are done; the warp owns the tensor memory.  Warps 2..5:
//    epilogue (tcgen05.ld of the accumulator, fp16 stores).  FUSED: warps 6..13 dequantize
//    (one 16-column tile of the 128 rows each), warp 14 copies the codes.
//  * Two accumulators of BN fp32 columns in tensor memory: the epilogue of one tile
//    overlaps the MMAs of the next.
//  * Every mbarrier wait first tests the phase inline; one that has to wait is bounded in
//    time (100 ms; a healthy one takes microseconds).  One that runs out sets a flag in a
//    device error word (qlinear_prefill_read_error) and a CTA-wide abort flag; every role
//    then leaves its loop, waits briefly for its copies and MMAs in flight, and the CTA
//    releases its tensor memory and exits.  A lost copy gives wrong numbers, never a hung
//    GPU.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdlib>
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

template <int BN, bool FUSED, int FMT = kW4, bool PAIR = false>
struct TcCfg {
  static_assert(BN == 128 || BN == 256, "token tile");
  // PAIR: a cluster of two CTAs on two SMs computes one tile of 2 x 128 weight rows with
  // tcgen05.mma.cta_group::2: each CTA holds its 128 rows of A and half of the tile's rows
  // of x in its own shared memory, and its 128 rows of the accumulator in its tensor memory.
  static constexpr int kCtas = PAIR ? 2 : 1;
  static constexpr int kRows = kBM * kCtas;                  // weight rows per tile (MMA M)
  static constexpr int kBRows = BN / kCtas;                  // rows of x one CTA copies
  static constexpr int kABytes = kBM * kBK * 2;              // 16 KB
  static constexpr int kBBytes = kBRows * kBK * 2;           // 8 .. 32 KB
  // FUSED: the stage's packed codes, as bulk-copied: per 16-row tile the half chunk of the
  // stage's 64 k (W4, LUT4: quad h, 512 B; W8: quads 2h, 2h + 1, 1 KB; W2: the whole 512-B
  // chunk, whose halves interleave per lane), then the block's parameters for the group
  // (scales and zeros 8 x 32 B each; LUT4: absmax 8 x 128 B)
  static constexpr int kCodeChunk = FMT == kW8 ? 1024 : 512;
  static constexpr int kCodeBytes = FUSED ? 8 * kCodeChunk : 0;
  static constexpr int kParChunk = FMT == kLUT4 ? 128 : 32;  // per tile, per array
  static constexpr int kParBytes = FUSED ? (FMT == kLUT4 ? 8 * 128 : 2 * 8 * 32) : 0;
  // A and B of one stage; FUSED: the codes and parameters of a stage live in a ring of their
  // own (SC slots), which a producer warp fills ahead of the A / B ring: a code slot is free
  // again as soon as the dequantizing warps have read it, long before the MMAs are done
  // with the stage, so the codes' HBM latency is covered by SC stages instead of S
  static constexpr int kStageBytes = kABytes + kBBytes;      // multiple of 1024
  static constexpr int kCodeSlot = (kCodeBytes + kParBytes + 127) / 128 * 128;
  static constexpr int kParOff = kCodeBytes;                 // inside a code slot
  static constexpr int kBudget = 232448 - 2048;              // bytes for the two rings
  // stages: as many as fit up to 8; FUSED: the most (up to 6) that leave six code slots
  static constexpr int pick_s() {
    if (!FUSED) return kBudget / kStageBytes < 8 ? kBudget / kStageBytes : 8;
    for (int st = 6; st >= 3; --st)
      if (kBudget - st * kStageBytes >= 6 * kCodeSlot) return st;
    return 2;
  }
  static constexpr int S = pick_s();
  static constexpr int SC0 = FUSED ? (kBudget - S * kStageBytes) / kCodeSlot : 0;
  static constexpr int SC = SC0 < 8 ? SC0 : 8;
  static constexpr int kCodeRingOff = S * kStageBytes;
  static_assert(S >= 3 && (!FUSED || SC >= 6), "pipeline depth");
  static constexpr int kEpiWarp0 = 2, kEpiWarps = 4;
  static constexpr int kDqWarp0 = kEpiWarp0 + kEpiWarps;
  static constexpr int kCodeWarp = kDqWarp0 + kDqWarps;      // FUSED: the code producer
  static constexpr int kWarps = FUSED ? kCodeWarp + 1 : kDqWarp0;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kBarOff = kCodeRingOff + SC * kCodeSlot;
  // full[S] empty[S] accf[2] acce[2] fin cfull[SC] cempty[SC]
  static constexpr int kSlotOff = kBarOff + 8 * (2 * S + 5 + 2 * SC);  // tmem base, abort flag
  static constexpr int kSmemBytes = kSlotOff + 16 + 1024;    // + slack to align the ring
  static constexpr uint32_t kTmemCols = 2 * BN;
  // full[s] (the leader CTA's, for both CTAs of a pair) completes on the TMA bytes of x (and
  // W) of every CTA of the tile plus one arrival per dequantizing warp; cfull[s] (FUSED, each
  // CTA its own) on the bytes of the stage's codes and parameters
  static constexpr uint32_t kFullCount = 1 + (FUSED ? kCtas * kDqWarps : 0);
  static constexpr uint32_t kFullBytes = kCtas * (kBBytes + (FUSED ? 0 : kABytes));
  static constexpr uint32_t kAccEmptyCount = kCtas * kEpiWarps;  // acce[a], the leader's
  static_assert(kSmemBytes + 64 <= 232448, "shared memory");
};

struct TcParams {
  const uint8_t* qw;     // FUSED: packed codes
  const void* p0;        // FUSED: packed scales | lut16
  const void* p1;        // FUSED: packed zeros | packed absmax
  __half* y;             // [M][N]
  float* partials;       // stream-K: fp32 partial tiles, two slots per CTA (null: whole tiles)
  uint32_t* counters;    // stream-K: arrivals per (tile, CTA of the tile, epilogue warp)
  int M, N, K, G, ntiles, mtiles, tiles;
  bool pair;             // host: launch the cluster-pair instance
};

// The k-block work of a CTA as a sequence of segments (tile t, k-blocks [kb0, kb1)).
//  * whole tiles (no partials): tiles c, c + C, c + 2C, ... each from k-block 0 to KB;
//  * stream-K: the flattened (tile, k-block) units [c U / C, (c + 1) U / C), U = tiles x KB,
//    cut at tile boundaries: only a CTA's first and last segments can be partial tiles,
//    and every CTA gets the same number of k-blocks to within one.
// A worker is a CTA, or a cluster pair of CTAs (both follow the same sequence).
struct SegIter {
  long long u, u1;  // stream-K: next unit, end of the range
  int j;            // whole tiles: next tile of this worker
  int w, W;         // this worker, number of workers
  __device__ void init(const TcParams& P, int KB, int w_, int W_) {
    w = w_;
    W = W_;
    const long long U = (long long)P.tiles * KB;
    u = w * U / W;
    u1 = (w + 1) * U / W;
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
    t = w + j * W;
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

// PAIR: the ::2 forms, executed by the same warp of both CTAs (the columns are taken in
// both tensor memories)
template <bool PAIR>
__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
  if constexpr (PAIR) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  } else {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
}
template <bool PAIR>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  if constexpr (PAIR)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` (a shared::cluster address: this CTA's, or the peer's) once every
// tcgen05.mma this thread issued before has completed.
template <bool PAIR>
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  if constexpr (PAIR)
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
  else
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// D[tmem] (+)= A[smem] . B[smem]^T, both K-major (shape in the instruction descriptor).
// PAIR: issued by the leader CTA; A's rows and B's rows come half from each CTA's shared
// memory (same offsets), D's rows half into each CTA's tensor memory.
template <bool PAIR>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  if constexpr (PAIR)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u)
        : "memory");
}
// This CTA's rank in its cluster; the shared::cluster address of this CTA's shared-memory
// address `a` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_addr(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
// Arrive on an mbarrier of another CTA of the cluster (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
// Every thread of every CTA of the cluster.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
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
// The same copy into this CTA's shared memory, its bytes completing on `bar` in either CTA
// of the pair (a shared::cluster address: the leader's barrier).
__device__ __forceinline__ void tma_2d_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
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
// and *abort, and returns false.  Every role leaves its loop on the first failed wait, so a
// broken pipeline ends the kernel within a few limits instead of one limit per remaining
// wait.  `cluster`: the phase completes on arrivals from the other CTA of a pair (acquire at
// cluster scope).
constexpr uint64_t kWaitNs = 100ull * 1000 * 1000;

// Non-blocking test of the phase (the fast path: the phase has usually completed already).
__device__ __forceinline__ bool mbar_ready(uint32_t bar, uint32_t parity, bool cluster) {
  uint32_t done;
  if (cluster)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
  return done != 0;
}

__device__ __noinline__ bool tc_wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                          uint32_t bit, uint64_t limit_ns, bool honor_abort,
                                          bool patient, uint32_t backoff_ns, bool cluster) {
  // The first kSpin rounds poll, sleeping backoff_ns between polls (the pipeline's waits are
  // usually short; the sleep keeps a polling lane from taking the issue slots of the warps
  // that do the work); after that each try_wait may suspend the thread for up to kSuspendNs
  // until the phase completes.  `patient` waiters (the epilogue, whose waits last a whole
  // tile) suspend from the start.  The clock is read only every 64 rounds.
  constexpr uint32_t kSpin = 2048, kSuspendNs = 500;
  uint64_t t0 = 0;
  for (uint32_t it = patient ? kSpin : 0;; ++it) {
    uint32_t done;
    if (cluster) {
      asm volatile(
          "{\n\t.reg .pred p;\n\t"
          "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(done)
          : "r"(bar), "r"(parity)
          : "memory");
    } else if (it < kSpin) {
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
      if (honor_abort && *abort) break;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0)
        t0 = now;
      else if (now - t0 > limit_ns)
        break;
    }
  }
  atomicOr(&g_tc_err, bit);
  *abort = 1u;
  return false;
}

__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                        uint32_t bit, uint64_t limit_ns = kWaitNs,
                                        bool honor_abort = true, bool patient = false,
                                        uint32_t backoff_ns = 0, bool cluster = false) {
  if (mbar_ready(bar, parity, cluster)) return true;
  return tc_wait_slow(bar, parity, abort, bit, limit_ns, honor_abort, patient, backoff_ns, cluster);
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

// The stage's codes and parameters of tile jj, from shared memory (tensor-copied by the code
// producer; layouts as in TcCfg): `cs` = the stage's code slot, `half` = kb % 2.
template <int FMT, class C>
__device__ __forceinline__ void dq_load_smem(uint32_t cs, int jj, int half, int lane,
                                             DqFrag<FMT>& f) {
  const int gi = lane >> 2;
  const uint32_t c = cs + jj * C::kCodeChunk;
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
  const uint32_t pa = cs + C::kParOff;
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

template <int BN, bool FUSED, int FMT, bool PAIR>
__global__ void __launch_bounds__(TcCfg<BN, FUSED, FMT, PAIR>::kThreads, 1)
    prefill_tc_kernel(const TcParams P, const __grid_constant__ CUtensorMap xmap,
                      const __grid_constant__ CUtensorMap wmap,
                      const __grid_constant__ CodeMaps cmaps) {
  using C = TcCfg<BN, FUSED, FMT, PAIR>;
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
  auto cfull = [&](int c) { return bars + 8 * (2 * C::S + 5 + c); };  // FUSED: codes landed
  auto cempty = [&](int c) { return bars + 8 * (2 * C::S + 5 + C::SC + c); };  // ... read
  const uint32_t slot = ring + C::kSlotOff;
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + C::kSlotOff + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = P.K / kBK;
  // PAIR: rank 0 (the leader) issues the MMAs and owns the barriers of the pair's pipeline
  // (full, acce); both CTAs copy their own halves of x (and W) and dequantize their own A
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int wk = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // worker
  const int nwk = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  // the leader's barrier `b` as this CTA addresses it; the peer's copy of own barrier `b`
  auto lead = [&](uint32_t b) { return (PAIR && !leader) ? cluster_addr(b, 0) : b; };
  auto arrive_lead = [&](uint32_t b) {
    if (PAIR && !leader)
      mbar_arrive_remote(cluster_addr(b, 0));
    else
      qlk::mbar_arrive(b);
  };
  // the leader's commits release both CTAs' barriers
  auto commit_both = [&](uint32_t b) {
    tc_commit<PAIR>(b);
    if constexpr (PAIR) tc_commit<PAIR>(cluster_addr(b, 1));
  };

  __shared__ float lut_s[16];
  if (FUSED && FMT == kLUT4 && threadIdx.x < 16)
    lut_s[threadIdx.x] = __half2float(static_cast<const __half*>(P.p0)[threadIdx.x]);
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::S; ++s) {
      qlk::mbar_init(full(s), C::kFullCount);
      qlk::mbar_init(empty(s), 1);
    }
    for (int c = 0; c < C::SC; ++c) {
      qlk::mbar_init(cfull(c), 1);
      qlk::mbar_init(cempty(c), kDqWarps);
    }
    for (int a = 0; a < 2; ++a) {
      qlk::mbar_init(accf(a), 1);
      qlk::mbar_init(acce(a), C::kAccEmptyCount);
    }
    qlk::mbar_init(fin, 1);
    *abort = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc<PAIR>(slot, C::kTmemCols);
  tc_fence_before();
  // the peer's copies and arrivals reach the leader's barriers only once they are set up
  if constexpr (PAIR)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::kSlotOff);

  if (warp == 0) {
    // ---- TMA producer (each CTA its own halves)
    if (lane == 0) {
      int it = 0, t, kb0, kb1;
      bool ok = true;
      SegIter sg;
      sg.init(P, KB, wk, nwk);
      while (ok && sg.next(P, KB, t, kb0, kb1)) {
        const int nt = t / P.mtiles, mt = t - nt * P.mtiles;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % C::S;
          if (it >= C::S &&
              !(ok = tc_wait(empty(s), ((it / C::S) - 1) & 1, abort, kErrStage, kWaitNs, true,
                             false, 64)))
            break;
          const uint32_t st = ring + s * C::kStageBytes;
          if (leader) qlk::mbar_arrive_expect_tx(full(s), C::kFullBytes);
          const int xrow = mt * BN + (int)rank * C::kBRows;
          const int wrow = nt * C::kRows + (int)rank * kBM;
          if constexpr (PAIR) {
            tma_2d_pair(st + C::kABytes, &xmap, kb * kBK, xrow, lead(full(s)));
            if constexpr (!FUSED) tma_2d_pair(st, &wmap, kb * kBK, wrow, lead(full(s)));
          } else {
            tma_2d(st + C::kABytes, &xmap, kb * kBK, xrow, full(s));
            if constexpr (!FUSED) tma_2d(st, &wmap, kb * kBK, wrow, full(s));
          }
        }
      }
      // no copy of this CTA is still in flight when it exits: wait for the last stages filled
      // (the leader's full barriers count the bytes of both CTAs of a pair; the pair meets
      // at a cluster barrier before either exits)
      if (leader)
        for (int i = (it > C::S ? it - C::S : 0); i < it; ++i)
          tc_wait(full(i % C::S), (i / C::S) & 1, abort, kErrStage, kWaitNs / 10, false);
    }
  } else if (FUSED && warp == C::kCodeWarp) {
    // ---- code producer: the stages' packed codes (rows: the block's 8 chunks of the group,
    // columns: the stage's half, or all of a W2 chunk) and the group's parameters, three
    // tensor copies per stage into the code ring; rows past the block are another group's
    // (unused) or read as zeros
    if (lane == 0) {
      int it = 0, t, kb0, kb1;
      bool ok = true;
      SegIter sg;
      sg.init(P, KB, wk, nwk);
      while (ok && sg.next(P, KB, t, kb0, kb1)) {
        const int nt = t / P.mtiles;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int c = it % C::SC;
          if (it >= C::SC &&
              !(ok = tc_wait(cempty(c), ((it / C::SC) - 1) & 1, abort, kErrStage, kWaitNs, true,
                             false, 64)))
            break;
          const uint32_t cs = ring + C::kCodeRingOff + c * C::kCodeSlot;
          const int g = kb >> 1, half = kb & 1;
          const int ch0 = (int)chunk_index(nt * C::kCtas + (int)rank, g, 0, P.G, P.ntiles);
          qlk::mbar_arrive_expect_tx(cfull(c), C::kCodeBytes + C::kParBytes);
          tma_2d(cs, &cmaps.codes, FMT == kW2 ? 0 : half * (C::kCodeChunk / 4), ch0, cfull(c));
          if constexpr (FMT == kLUT4) {
            tma_2d(cs + C::kParOff, &cmaps.p1, 0, ch0, cfull(c));
          } else {
            tma_2d(cs + C::kParOff, &cmaps.p0, 0, ch0, cfull(c));
            tma_2d(cs + C::kParOff + 8 * 32, &cmaps.p1, 0, ch0, cfull(c));
          }
        }
      }
      // no copy in flight when the CTA exits
      for (int i = (it > C::SC ? it - C::SC : 0); i < it; ++i)
        tc_wait(cfull(i % C::SC), (i / C::SC) & 1, abort, kErrStage, kWaitNs / 10, false);
    }
  } else if (warp == 1) {
    // ---- MMA issuer (the leader of a pair)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_f16(C::kRows, BN);
      int it = 0, j = 0, t, kb0, kb1;
      bool ok = true;
      SegIter sg;
      sg.init(P, KB, wk, nwk);
      for (; ok && sg.next(P, KB, t, kb0, kb1); ++j) {
        const int a = j & 1;
        if (j >= 2 &&
            !(ok = tc_wait(acce(a), ((j >> 1) - 1) & 1, abort, kErrAcc, kWaitNs, true, false, 0, PAIR)))
          break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * BN);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % C::S;
          if (!(ok = tc_wait(full(s), (it / C::S) & 1, abort, kErrStage, kWaitNs, true, false, 32,
                             PAIR && FUSED)))
            break;
          tc_fence_after();
          const uint32_t st = ring + s * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma<PAIR>(d, desc_sw128(st + 32 * kk), desc_sw128(st + C::kABytes + 32 * kk), idesc,
                         (kb != kb0) || (kk != 0));
          commit_both(empty(s));  // the stage is free once these MMAs have read it
        }
        if (ok) commit_both(accf(a));  // the segment's accumulator is complete
      }
      // every MMA issued has completed before the tensor memory is released (the peer
      // releases its columns after the cluster barrier below, which the leader reaches
      // only after this wait)
      tc_commit<PAIR>(fin);
      tc_wait(fin, 0, abort, kErrAcc, kWaitNs / 10, false);
    }
  } else if (warp < C::kDqWarp0) {
    // ---- epilogue: warp w reads accumulator lanes 32 (w % 4) .. + 31 (this CTA's weight rows)
    const int q = warp & 3;
    const long long U = (long long)P.tiles * KB;
    int j = 0, t, kb0, kb1;
    SegIter sg;
    sg.init(P, KB, wk, nwk);
    for (; sg.next(P, KB, t, kb0, kb1); ++j) {
      const int a = j & 1;
      const int nt = t / P.mtiles, mt = t - nt * P.mtiles;
      bool ok = true;
      if (lane == 0) ok = tc_wait(accf(a), (j >> 1) & 1, abort, kErrAcc, kWaitNs, true, true);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after();
      const int row = 32 * q + lane;
      const int n = nt * C::kRows + (int)rank * kBM + row;
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
        if (lane == 0) arrive_lead(acce(a));
        continue;
      }
      // part of a tile (stream-K): publish this CTA's fp32 partial; the last contributor
      // adds all of them in worker order and stores y (nobody waits for anybody)
      const int pslot = 2 * (int)blockIdx.x + (j == 0 ? 0 : 1);
      float* mine = P.partials + ((size_t)pslot * kBM + row) * BN;
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
      if (lane == 0) arrive_lead(acce(a));  // the accumulator is free again
      const int cf = sk_cta_of((long long)t * KB, U, nwk);
      const int cl = sk_cta_of((long long)(t + 1) * KB - 1, U, nwk);
      uint32_t* counter = P.counters + ((size_t)t * C::kCtas + rank) * 4 + q;
      uint32_t prev = 0;
      if (lane == 0) prev = qlk::arrive_acq_rel(counter);
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev + 1 != (uint32_t)(cl - cf + 1)) continue;
      __syncwarp();
      for (int c0 = 0; c0 < cols; c0 += 16) {
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
        for (int cc = cf; cc <= cl; ++cc) {
          const int cta = cc * C::kCtas + (int)rank;
          const int sl = (sk_begin(cc, U, nwk) >= (long long)t * KB) ? 2 * cta : 2 * cta + 1;
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
      if (lane == 0) *counter = 0u;  // ready for the next call
    }
  } else if constexpr (FUSED) {
    // ---- dequantizing producers: warp dw fills rows 16 dw .. 16 dw + 15 of this CTA's A of
    // stage s (once the MMAs are done with it) from the codes in code slot c, then releases
    // both
    const int dw = warp - C::kDqWarp0;
    int it = 0, t, kb0, kb1;
    bool ok = true;
    SegIter sg;
    sg.init(P, KB, wk, nwk);
    while (ok && sg.next(P, KB, t, kb0, kb1)) {
      // tiles of this CTA's 128-row block (none for a block past N)
      const int blk = (t / P.mtiles) * C::kCtas + (int)rank;
      const int tb = blk * kBlockTiles < P.ntiles ? tiles_in_block(blk, P.ntiles) : 0;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const int s = it % C::S, c = it % C::SC;
        if (lane == 0) {
          ok = tc_wait(cfull(c), (it / C::SC) & 1, abort, kErrStage, kWaitNs, true, false, 32);
          if (ok && it >= C::S)
            ok = tc_wait(empty(s), ((it / C::S) - 1) & 1, abort, kErrStage, kWaitNs, true, false, 32);
        }
        if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
        const uint32_t st = ring + s * C::kStageBytes;
        DqFrag<FMT> f;
        if (dw < tb) dq_load_smem<FMT, C>(ring + C::kCodeRingOff + c * C::kCodeSlot, dw, kb & 1, lane, f);
        if (dw < tb) dq_store<FMT>(f, st, dw, lane, lut_s);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the MMAs
        __syncwarp();
        // the code slot is released only now, once every lane has used the words it read
        // (releasing it right after the shared loads and a __syncwarp let the next copy
        // overwrite words some lanes had not yet read: wrong results in a stress run)
        if (lane == 0) {
          qlk::mbar_arrive(cempty(c));
          arrive_lead(full(s));
        }
      }
    }
  }

  tc_fence_before();
  // PAIR: neither CTA exits (or releases its tensor memory) while the other may still
  // arrive on its barriers or the leader's MMAs may still use its memory
  if constexpr (PAIR)
    cluster_sync();
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<PAIR>(tmem, C::kTmemCols);
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

// Workers (CTAs, or cluster pairs) that are resident at once on this device, per instance.
template <int BN, bool FUSED, int FMT, bool PAIR>
int resident_workers(int dev, int sms) {
  using C = TcCfg<BN, FUSED, FMT, PAIR>;
  auto fn = prefill_tc_kernel<BN, FUSED, FMT, PAIR>;
  static std::mutex mu;
  static std::unordered_map<int, int> known;
  std::lock_guard<std::mutex> lk(mu);
  auto k = known.find(dev);
  if (k != known.end()) return k->second;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
      cudaSuccess)
    return 0;
  int n = 0;
  if constexpr (PAIR) {
    // pairs must sit on two SMs of one GPC: count the clusters that fit, not SMs / 2
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) n = 0;
  } else {
    int occ = 0;  // the CTA (threads x registers, shared memory) must fit on an SM
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, C::kThreads, C::kSmemBytes) ==
            cudaSuccess &&
        occ >= 1)
      n = sms;
  }
  if (n > 0) known[dev] = n;
  return n;
}

template <int BN, bool FUSED, int FMT, bool PAIR>
ql_status launch_tc(const TcParams& P, const void* x, const void* w, cudaStream_t st) {
  using C = TcCfg<BN, FUSED, FMT, PAIR>;
  auto fn = prefill_tc_kernel<BN, FUSED, FMT, PAIR>;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QL_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return QL_ERR_CUDA;
  const int maxw = resident_workers<BN, FUSED, FMT, PAIR>(dev, sms);
  if (maxw <= 0) return QL_ERR_CUDA;
  CUtensorMap xmap, wmap;
  CodeMaps cm;
  if (!encode_kmajor(&xmap, x, P.M, P.K, C::kBRows)) return QL_ERR_CUDA;
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
  // stream-K: one worker per SM (pair of SMs), at most one per k-block, so that every worker
  // has work (the fix-up counts the workers whose ranges meet a tile), the k-blocks shared out
  // evenly; whole tiles: at most one worker per tile
  const long long units = P.partials ? (long long)P.tiles * (P.K / kBK) : P.tiles;
  const int workers = units < maxw ? (int)units : maxw;
  if constexpr (PAIR) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * workers, 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = st;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fn, P, xmap, wmap, cm) != cudaSuccess) return QL_ERR_CUDA;
  } else {
    fn<<<workers, C::kThreads, C::kSmemBytes, st>>>(P, xmap, wmap, cm);
  }
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

// Tile form: the dense GEMM on cluster pairs (tcgen05 cta_group::2: each CTA copies half of
// the tile's x, which the dense GEMM's L2 traffic and power budget favour), the fused one on
// single CTAs (its dequantizing warps would otherwise also wait for the other CTA's).  Both
// measured on 8192 x 28672 at M = 512 and 2048.  QLINEAR_TC_PAIR = 0 / 1 forces one form.
bool use_pair(bool fused) {
  const char* e = getenv("QLINEAR_TC_PAIR");
  if (e && (e[0] == '0' || e[0] == '1')) return e[0] == '1';
  return !fused;
}

template <bool FUSED, int FMT>
ql_status launch_bn(const TcParams& P, const void* x, const void* w, cudaStream_t st) {
  if (P.pair)
    return P.M <= 128 ? launch_tc<128, FUSED, FMT, true>(P, x, w, st)
                      : launch_tc<256, FUSED, FMT, true>(P, x, w, st);
  return P.M <= 128 ? launch_tc<128, FUSED, FMT, false>(P, x, w, st)
                    : launch_tc<256, FUSED, FMT, false>(P, x, w, st);
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
  P.pair = use_pair(packed != nullptr);
  const int bn = M <= 128 ? 128 : 256;
  const int rows = P.pair ? 2 * kBM : kBM;
  P.mtiles = (M + bn - 1) / bn;
  P.tiles = ((N + rows - 1) / rows) * P.mtiles;
  P.partials = nullptr;
  P.counters = nullptr;
  return P;
}

// Workspace of the stream-K schedule: arrival counters (one per tile, CTA of the tile and
// epilogue warp; zero between calls; sized for 256-row tiles of two CTAs, which is at least
// the count for 128-row tiles) and two fp32 partial tiles (128 x BN) per CTA.
struct SkLayout {
  size_t counter_bytes, partial_offset, bytes;
};
SkLayout sk_layout(int M, int N, int sms) {
  const int bn = M <= 128 ? 128 : 256;
  const long long tiles = (long long)((N + 2 * kBM - 1) / (2 * kBM)) * 2 * ((M + bn - 1) / bn);
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
