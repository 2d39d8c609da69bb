// C ABI of the quantized GEMV library: argument checks, launch planning, kernel
// instances and the debug decode kernels.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <atomic>
#include <mutex>
#include <unordered_map>

#include "kernels.cuh"
#include "policy.h"
#include "qlinear.h"

using namespace qlayout;

namespace {

constexpr int kMaxCtasPerSm = 8;
constexpr size_t kErrBytes = 256;  // workspace[0..255]: error word (first 4 bytes)

// Settings of qlinear_debug_wait_test (tests of the bounded waits; defaults otherwise).
std::atomic<uint32_t> g_wait_limit{qlk::kSpinLimit};
std::atomic<uint32_t> g_test_us{0};

bool fmt_ok(int fmt) {
  return fmt == kW2 || fmt == kW3 || fmt == kW4 || fmt == kW8 || fmt == kLUT4;
}
// ... and the formats the GEMV (plan, workspace) also serves: the tensor-core codebook layout
bool gemv_fmt_ok(int fmt) { return fmt_ok(fmt) || fmt == kCB; }
bool aligned(const void* p, size_t a) { return ((uintptr_t)p & (a - 1)) == 0; }
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Plan {
  int C;            // CTAs
  long long U;      // units
  int nblocks, ntiles, G, MT, WPU, NC, T, threads, smem;
  bool M1;          // W4 with one row of x: the kernel keeps only batch column 0
  bool OCC2;        // ... with registers for two CTAs per SM (grids of at most 2 per SM)
  int NS;           // quantization sub-groups per 128-k unit (group 128 / NS)
  size_t counter_offset, partial_offset, ws_bytes;
};

struct KernelInfo {
  const void* fn;  // qgemv_kernel<...>: its second parameter a tensor map of x if xt
  int threads, smem, NC, T;
  bool xt;
};

template <int FMT, int MT, bool OUTL, int WPU = qlk::default_wpu(FMT, MT), bool M1 = false,
          int OCC = 0, int NS = 1, bool TH = false>
KernelInfo kernel_info() {
  using C = qlk::Cfg<FMT, MT, OUTL, WPU, M1, OCC, NS>;
  return KernelInfo{
      reinterpret_cast<const void*>(qlk::qgemv_kernel<FMT, MT, OUTL, WPU, M1, OCC, NS, TH>),
      C::kThreads, C::kSmemBytes, C::NC, C::T, !M1};
}

// Instances with the test hooks of the bounded waits (same shared memory and threads as the
// instance they stand in for): W4 with one row of x (three and two CTAs per SM) and W4 at
// M = 9..16.  Other kernels run without the hooks.
bool test_kernel(int fmt, int MT, bool outl, int wpu, bool m1, bool occ2, int ns, KernelInfo* k) {
  if (fmt != kW4 || outl || ns != 1) return false;
  if (MT == 2) {
    *k = kernel_info<kW4, 2, false, 2, false, 0, 1, true>();
    return true;
  }
  if (m1 && wpu == 1) {
    *k = occ2 ? kernel_info<kW4, 1, false, 1, true, 2, 1, true>()
              : kernel_info<kW4, 1, false, 1, true, 0, 1, true>();
    return true;
  }
  return false;
}

// Finer quantization groups (NS sub-groups per 128-k unit): two warps per unit for every
// format, so each warp holds two quads of two tiles (the sub-groups' scale and zero pairs
// take registers that four tiles at a time would not leave).
constexpr int kFineWpu = 2;

template <int FMT, int NS>
KernelInfo fine_kernel(int MT, bool m1) {
  if (MT == 2) return kernel_info<FMT, 2, false, kFineWpu, false, 0, NS>();
  return m1 ? kernel_info<FMT, 1, false, kFineWpu, true, 0, NS>()
            : kernel_info<FMT, 1, false, kFineWpu, false, 0, NS>();
}

template <int NS>
KernelInfo fine_kernel_fmt(int fmt, int MT, bool m1) {
  switch (fmt) {
    case kW2: return fine_kernel<kW2, NS>(MT, m1);
    case kW8: return fine_kernel<kW8, NS>(MT, m1);
    default: return fine_kernel<kW4, NS>(MT, m1);
  }
}

// The M <= 8 kernel of a format: its single-row variant for M = 1, else the one for M >= 2.
template <int FMT, bool OUTL>
KernelInfo m8_kernel(bool m1) {
  return m1 ? kernel_info<FMT, 1, OUTL, qlk::default_wpu(FMT, 1), true>()
            : kernel_info<FMT, 1, OUTL>();
}

// wpu: warps per unit; W4 at M <= 8 has the one-warp default and 2- and 4-warp variants for
// small layers, every other kernel its default only.  m1: W4 with exactly one row of x.
// occ2: the one-warp M = 1 kernel with registers for two CTAs per SM instead of three.
template <int WPU>
KernelInfo w4_m8_kernel(bool m1) {
  return m1 ? kernel_info<kW4, 1, false, WPU, true>() : kernel_info<kW4, 1, false, WPU, false>();
}

KernelInfo select_kernel(int fmt, int MT, bool outl, int wpu, bool m1, bool occ2 = false,
                         int ns = 1) {
  if (ns == 2) return fine_kernel_fmt<2>(fmt, MT, m1);
  if (ns == 4) return fine_kernel_fmt<4>(fmt, MT, m1);
  if (occ2 && fmt == kW4 && MT == 1 && !outl && wpu == 1 && m1)
    return kernel_info<kW4, 1, false, 1, true, 2>();
  if (outl) return MT == 1 ? m8_kernel<kW4, true>(m1) : kernel_info<kW4, 2, true>();
  switch (fmt) {
    case kW2: return MT == 1 ? m8_kernel<kW2, false>(m1) : kernel_info<kW2, 2, false>();
    case kW3: return MT == 1 ? m8_kernel<kW3, false>(m1) : kernel_info<kW3, 2, false>();
    case kW4:
      if (MT == 2) return kernel_info<kW4, 2, false>();
      return wpu == 4 ? w4_m8_kernel<4>(m1) : wpu == 2 ? w4_m8_kernel<2>(m1) : w4_m8_kernel<1>(m1);
    case kW8: return MT == 1 ? m8_kernel<kW8, false>(m1) : kernel_info<kW8, 2, false>();
    case kCB: return MT == 1 ? m8_kernel<kCB, false>(m1) : kernel_info<kCB, 2, false>();
    default: return MT == 1 ? m8_kernel<kLUT4, false>(m1) : kernel_info<kLUT4, 2, false>();
  }
}

// Opt a kernel into its dynamic shared memory and query its resident CTAs per SM
// (once per kernel and device, then cached).
cudaError_t prepare_kernel(const KernelInfo& k, int dev, int* ctas) {
  static std::mutex mu;
  static std::unordered_map<uint64_t, int> cache;
  const uint64_t key = ((uint64_t)(uintptr_t)k.fn << 8) ^ (uint64_t)dev;
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *ctas = it->second;
    return cudaSuccess;
  }
  cudaError_t e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k.fn, k.threads, k.smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) occ = 1;
  if (occ > kMaxCtasPerSm) occ = kMaxCtasPerSm;
  cache[key] = occ;
  *ctas = occ;
  return cudaSuccess;
}

cudaError_t make_plan(int fmt, int M, int N, int K, bool outl, Plan* p, int ns = 1) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  p->MT = M <= 8 ? 1 : 2;
  p->WPU = ns > 1 ? kFineWpu : qlk::default_wpu(fmt, p->MT);
  p->M1 = M == 1;
  p->OCC2 = false;
  p->NS = ns;
  const KernelInfo k = select_kernel(fmt, p->MT, outl, p->WPU, p->M1, false, ns);
  int occ = 1;
  e = prepare_kernel(k, dev, &occ);
  if (e != cudaSuccess) return e;
  p->NC = k.NC;
  p->T = k.T;
  p->threads = k.threads;
  p->smem = k.smem;
  p->G = K / kGroup;
  p->ntiles = N / kTileN;
  p->nblocks = (p->ntiles + kBlockTiles - 1) / kBlockTiles;
  p->U = (long long)p->nblocks * p->G;
  const long long slots = (long long)sms * occ;  // CTAs resident at once
  long long C = slots;
  // Small layers (latency-bound: at most 16 units per CTA) use a block-aligned split when it
  // fills most of the GPU: k CTAs per 128-column block with k | G gives every CTA a
  // whole-group slice of one block, so each block has exactly k partial sums and no CTA
  // straddles two blocks.  Larger layers stream over all resident slots (stream-K).
  for (long long k = p->G; k >= 1; --k) {
    if (p->G % k == 0 && p->nblocks * k <= slots) {
      const long long ca = p->nblocks * k;
      if (ca * 100 >= slots * 55 && p->U <= 16 * ca) C = ca;
      break;
    }
  }
  // W4 at M = 1 has a variant with registers for two CTAs per SM (fewer spills).  On small
  // layers a block-aligned grid of at most two CTAs per SM running it beats three:
  //  - the largest k | G with nblocks * k <= 2 SMs keeps every CTA's share of its block
  //    equal;
  //  - if that leaves over a fifth of the two-per-SM slots idle, take the most CTAs per
  //    block that fit instead: C = nblocks * k is still block-aligned, because CTA c covers
  //    units [c G / k, (c + 1) G / k) of block c / k.
  bool small_m1 = false;
  if (p->M1 && fmt == kW4 && !outl && ns == 1) {
    const long long c2 = 2LL * sms, kmax = c2 / p->nblocks;
    if (kmax >= 1 && p->U <= 16 * p->nblocks * kmax) {
      long long kd = kmax;
      while (p->G % kd) --kd;
      const long long k = (p->nblocks * kd * 5 >= c2 * 4) ? kd : kmax;
      C = p->nblocks * k;
      small_m1 = true;
    }
  }
  // a measured policy entry may fix the grid size and the warps per unit
  const qpolicy::Choice pol = qpolicy::lookup(fmt, outl, M, N, K);
  if (pol.ctas > 0) C = pol.ctas;
  // QLINEAR_MAX_CTAS forces the grid size (A/B runs, tests of the split-K fix-up)
  if (const char* cap = getenv("QLINEAR_MAX_CTAS")) {
    const long long v = atoll(cap);
    if (v > 0) C = v;
  }
  if (outl) {  // a CTA keeps the Tile-COO offsets of its units in shared memory
    const long long cmin = (p->U + qlk::kMaxUnitsPerCta - 1) / qlk::kMaxUnitsPerCta;
    if (C < cmin) C = cmin;
  }
  if (C > p->U) C = p->U;
  // the kernel's stream-K index arithmetic is 32-bit
  if (p->U * C >= (1LL << 31)) return cudaErrorInvalidValue;
  p->C = (int)C;
  // W4 at 2 <= M <= 8: a CTA with few units shares each unit among more warps, which
  // shortens the one unit a warp would otherwise work through alone.  The M = 1 kernel
  // (half the epilogue) is fastest with one warp per unit on every layer measured.
  // QLINEAR_WPU = 1, 2 or 4 overrides.
  if (fmt == kW4 && p->MT == 1 && !outl && ns == 1) {
    const long long per_cta = (p->U + C - 1) / C;
    int wpu = p->M1 ? 1 : per_cta <= 4 ? 4 : per_cta <= 24 ? 2 : 1;
    if (pol.wpu > 0) wpu = pol.wpu;
    if (const char* w = getenv("QLINEAR_WPU")) {
      const int v = atoi(w);
      if (v == 1 || v == 2 || v == 4) wpu = v;
    }
    if (wpu != p->WPU) {
      const KernelInfo k2 = select_kernel(fmt, p->MT, outl, wpu, p->M1);
      int occ2 = 1;
      e = prepare_kernel(k2, dev, &occ2);
      if (e != cudaSuccess) return e;
      if (occ2 >= occ) {  // never fewer resident CTAs than the grid was sized for
        p->WPU = wpu;
        p->threads = k2.threads;
        p->smem = k2.smem;
      }
    }
    // A grid of at most two CTAs per SM leaves the third slot empty: then the M = 1 kernel
    // with more registers per thread (fewer spills) is faster.
    if (p->M1 && p->WPU == 1 && (small_m1 || C <= 2LL * sms)) {
      const KernelInfo k3 = select_kernel(fmt, p->MT, outl, 1, true, true);
      int occ3 = 1;
      e = prepare_kernel(k3, dev, &occ3);
      if (e != cudaSuccess) return e;
      if ((long long)occ3 * sms >= C) {
        p->OCC2 = true;
        p->threads = k3.threads;
        p->smem = k3.smem;
      }
    }
  }
  p->counter_offset = kErrBytes;
  p->partial_offset = align_up(p->counter_offset + (size_t)p->nblocks * p->NC * sizeof(uint32_t), 256);
  p->ws_bytes = p->partial_offset +
                (size_t)2 * p->C * p->NC * p->T * 32 * 4 * p->MT * sizeof(float);
  return cudaSuccess;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no link
// against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// x [M][K] fp16 as a 2-D tensor (K innermost), box 128 x M: one copy brings a group's
// 128 elements of every row.  x is 16-byte aligned and the row stride 2K bytes a multiple of
// 256, as the copy requires.
bool encode_x_map(CUtensorMap* map, const void* x, int M, int K) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kGroup, (cuuint32_t)M};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(x), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool shape_ok(int M, int N, int K) {
  return M >= 1 && M <= 16 && N >= kTileN && K >= kGroup && N % kTileN == 0 && K % kGroup == 0;
}

struct Call {
  int fmt;
  bool outl;
  const void* x;
  const void* qw;
  const void* p0;
  const void* p1;
  const uint32_t* toff;
  const uint8_t* trc;
  const uint16_t* tval;
  void* y;
  int M, N, K;
  void* ws;
  size_t ws_bytes;
  cudaStream_t stream;
  int ns = 1;  // sub-groups per 128-k unit (from the group size)
};

// sub-groups per 128-k unit for a group size of the uniform formats: 4 (32), 2 (64),
// 1 (128, or per-channel g = K with the parameters repeated per unit by the packer)
int subgroups(int group, int K) {
  if (group == 32) return 4;
  if (group == 64) return 2;
  if (group == kGroup || group == K) return 1;
  return 0;
}

// Argument checks that need no device state (pointers, shapes, alignment).
ql_status check_call(const Call& c) {
  if (!c.x || !c.qw || !c.p0 || !c.p1 || !c.y) return QL_ERR_NULL;
  if (c.outl && (!c.toff || !c.trc || !c.tval)) return QL_ERR_NULL;
  if (!shape_ok(c.M, c.N, c.K)) return QL_ERR_SHAPE;
  if (c.outl && c.N % 128) return QL_ERR_SHAPE;
  if (!aligned(c.x, 16) || !aligned(c.qw, 32) || !aligned(c.y, 2)) return QL_ERR_ALIGN;
  // parameters arrive by bulk copies (16-byte aligned sources); the LUT and the codebook
  // are read directly
  if (c.fmt == kLUT4) {
    if (!aligned(c.p0, 2) || !aligned(c.p1, 16)) return QL_ERR_ALIGN;
  } else if (c.fmt == kCB) {
    if (!aligned(c.p0, 16) || !aligned(c.p1, 8)) return QL_ERR_ALIGN;
  } else if (!aligned(c.p0, 16) || !aligned(c.p1, 16)) {
    return QL_ERR_ALIGN;
  }
  if (c.outl && (!aligned(c.toff, 4) || !aligned(c.trc, 2) || !aligned(c.tval, 2)))
    return QL_ERR_ALIGN;
  return QL_OK;
}

ql_status run(const Call& c) {
  const ql_status chk = check_call(c);
  if (chk != QL_OK) return chk;
  Plan p;
  if (make_plan(c.fmt, c.M, c.N, c.K, c.outl, &p, c.ns) != cudaSuccess) return QL_ERR_CUDA;
  if (!c.ws || c.ws_bytes < p.ws_bytes) return QL_ERR_WORKSPACE;
  if (!aligned(c.ws, 16)) return QL_ERR_ALIGN;
  qlk::GemvParams P;
  P.x = static_cast<const __half*>(c.x);
  P.qw = static_cast<const uint8_t*>(c.qw);
  P.sc = static_cast<const __half*>(c.p0);
  P.zp = c.p1;
  P.tile_off = c.toff;
  P.tile_rc = reinterpret_cast<const uint16_t*>(c.trc);
  P.tile_val = c.tval;
  P.y = static_cast<__half*>(c.y);
  P.err = static_cast<uint32_t*>(c.ws);
  P.counters = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(c.ws) + p.counter_offset);
  P.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(c.ws) + p.partial_offset);
  P.M = c.M;
  P.N = c.N;
  P.K = c.K;
  P.G = p.G;
  P.nblocks = p.nblocks;
  P.ntiles = p.ntiles;
  P.U = (int)p.U;
  P.C = p.C;
  P.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
  P.test_us = g_test_us.load(std::memory_order_relaxed);
  KernelInfo k = select_kernel(c.fmt, p.MT, c.outl, p.WPU, p.M1, p.OCC2, p.NS);
  if (P.wait_limit != qlk::kSpinLimit || P.test_us != 0) {  // qlinear_debug_wait_test is active
    KernelInfo kt;
    if (test_kernel(c.fmt, p.MT, c.outl, p.WPU, p.M1, p.OCC2, p.NS, &kt)) {
      int dev = 0, occ = 0;
      if (cudaGetDevice(&dev) != cudaSuccess || prepare_kernel(kt, dev, &occ) != cudaSuccess)
        return QL_ERR_CUDA;
      k = kt;
    }
  }
  // Programmatic stream serialization: the kernel may start while the previous kernel in
  // the stream drains; it requests only static weight bytes before griddepcontrol.wait.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.C);
  cfg.blockDim = dim3((unsigned)k.threads);
  cfg.dynamicSmemBytes = (size_t)k.smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (k.xt) {
    CUtensorMap xmap;
    if (!encode_x_map(&xmap, c.x, c.M, c.K)) return QL_ERR_CUDA;
    void* args[2] = {&P, &xmap};
    if (cudaLaunchKernelExC(&cfg, k.fn, args) != cudaSuccess) return QL_ERR_CUDA;
  } else {
    qlk::NoXMap none{0};
    void* args[2] = {&P, &none};
    if (cudaLaunchKernelExC(&cfg, k.fn, args) != cudaSuccess) return QL_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// debug decode kernels: one warp per chunk, same fragment extraction as the GEMV

template <int FMT>
__device__ __forceinline__ uint32_t field_shift(int s, int r) {
  if constexpr (FMT == kW4) return (r & 1) ? 4u : 0u;
  if constexpr (FMT == kW2) return 4u * (s & 1) + ((r & 1) ? 2u : 0u);
  return 0u;
}

template <int FMT, bool DEQ>
__global__ void __launch_bounds__(128) debug_kernel(const uint8_t* packed, const void* p0,
                                                    const void* p1, uint8_t* codes, float* w,
                                                    int N, int K) {
  __shared__ uint32_t tbl[FMT == kLUT4 ? 256 * 32 : 1];
  const int G = K / kGroup, ntiles = N / kTileN;
  if constexpr (FMT == kLUT4 && DEQ) {
    qlk::build_lut_table(tbl, static_cast<const __half*>(p0), threadIdx.x, 128);
    __syncthreads();
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long id = (long long)blockIdx.x * 4 + warp;
  if (id >= (long long)ntiles * G) return;
  const int g = (int)(id % G), j = (int)(id / G);
  const int b = j / kBlockTiles, jj = j % kBlockTiles;
  const long long ch = chunk_index(b, g, jj, G, ntiles);
  constexpr int KW = qlk::Fmt<FMT>::kWords;
  uint32_t wv[KW];
  const uint32_t* src = reinterpret_cast<const uint32_t*>(packed + ch * chunk_bytes(FMT));
#pragma unroll
  for (int i = 0; i < KW; ++i) wv[i] = src[word_index_fmt(FMT, i, lane)];
  const int gi = lane >> 2, t4 = lane & 3;
  float2 s2 = make_float2(0.f, 0.f), z2 = s2;
  float4 am = make_float4(0.f, 0.f, 0.f, 0.f);
  if (DEQ) {
    if constexpr (FMT == kLUT4) {
      am = *reinterpret_cast<const float4*>(static_cast<const float*>(p1) + ch * 32 + gi * 4);
    } else {
      s2 = __half22float2(*reinterpret_cast<const __half2*>(static_cast<const __half*>(p0) + ch * 16 + gi * 2));
      z2 = __half22float2(*reinterpret_cast<const __half2*>(static_cast<const __half*>(p1) + ch * 16 + gi * 2));
    }
  }
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    uint32_t a[4];
    if constexpr (FMT == kLUT4) {
      if (DEQ) qlk::frag_lut(wv[s], (uint32_t)__cvta_generic_to_shared(tbl) + 4u * (uint32_t)lane, a);
      else a[0] = a[1] = a[2] = a[3] = 0u;
    } else {
      qlk::frag_uniform<(FMT == kW3) ? kW2 : FMT>(wv, s, a);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = gi + 8 * (r & 1);
        const int dk = e + 2 * (r >> 1);
        const int k = g * kGroup + k_in_group(s, t4, dk);
        const int n = j * kTileN + row;
        const __half hv = __ushort_as_half((unsigned short)(a[r] >> (16 * e)));
        if constexpr (FMT == kLUT4) {
          const uint32_t byte = (wv[s] >> (8 * r)) & 0xFFu;
          const uint32_t q = e ? (byte >> 4) : (byte & 0xFu);
          if (DEQ) {
            const float amv = (s >= 4) ? ((r & 1) ? am.w : am.z) : ((r & 1) ? am.y : am.x);
            w[(size_t)k * N + n] = __fmul_rn(__half2float(hv), amv);
          } else {
            codes[(size_t)k * N + n] = (uint8_t)q;
          }
        } else {
          // the fp16 value is code * 2^(shift - 24): decode it numerically
          const uint32_t iv = (uint32_t)(__half2float(hv) * 16777216.0f);
          uint32_t q = iv >> field_shift<(FMT == kW3) ? kW2 : FMT>(s, r);
          if constexpr (FMT == kW3)  // high bit: bit 4 (s % 4) + r of each half of word 4 + s / 4
            q |= ((wv[4 + (s >> 2)] >> (16 * e + 4 * (s & 3) + r)) & 1u) << 2;
          if (DEQ) {
            const float sc = (r & 1) ? s2.y : s2.x, zc = (r & 1) ? z2.y : z2.x;
            w[(size_t)k * N + n] = __fmul_rn(sc, (float)q - zc);
          } else {
            codes[(size_t)k * N + n] = (uint8_t)q;
          }
        }
      }
  }
}

template <bool DEQ>
ql_status launch_debug(int fmt, const void* packed, const void* p0, const void* p1,
                       uint8_t* codes, float* w, int N, int K, cudaStream_t st) {
  const long long chunks = (long long)(N / kTileN) * (K / kGroup);
  const unsigned grid = (unsigned)((chunks + 3) / 4);
  switch (fmt) {
    case kW2: debug_kernel<kW2, DEQ><<<grid, 128, 0, st>>>(static_cast<const uint8_t*>(packed), p0, p1, codes, w, N, K); break;
    case kW3: debug_kernel<kW3, DEQ><<<grid, 128, 0, st>>>(static_cast<const uint8_t*>(packed), p0, p1, codes, w, N, K); break;
    case kW4: debug_kernel<kW4, DEQ><<<grid, 128, 0, st>>>(static_cast<const uint8_t*>(packed), p0, p1, codes, w, N, K); break;
    case kW8: debug_kernel<kW8, DEQ><<<grid, 128, 0, st>>>(static_cast<const uint8_t*>(packed), p0, p1, codes, w, N, K); break;
    default: debug_kernel<kLUT4, DEQ><<<grid, 128, 0, st>>>(static_cast<const uint8_t*>(packed), p0, p1, codes, w, N, K); break;
  }
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

}  // namespace

// ---------------------------------------------------------------------------
// exported entry points

extern "C" const char* ql_status_str(int status) {
  switch (status) {
    case QL_OK: return "ok";
    case QL_ERR_NULL: return "null pointer argument";
    case QL_ERR_SHAPE: return "unsupported shape (M in 1..16, N % 16 == 0, K % 128 == 0, group 128 / 64 / 32 / K, block 64)";
    case QL_ERR_ALIGN: return "misaligned pointer";
    case QL_ERR_UNSUPPORTED: return "unknown format";
    case QL_ERR_WORKSPACE: return "workspace missing or too small";
    case QL_ERR_CUDA: return "CUDA error";
    case QL_ERR_LIBRARY: return "reserved (no library is opened at run time)";
    default: return "unknown status";
  }
}

extern "C" size_t qlinear_workspace_bytes(int fmt, int M, int N, int K) {
  if (!gemv_fmt_ok(fmt) || !shape_ok(M, N, K)) return 0;
  Plan p;
  if (make_plan(fmt, M, N, K, false, &p) != cudaSuccess) return 0;
  // the finer-group kernels (group 64, 32) may resolve to another occupancy: cover them
  if (fmt != kLUT4 && fmt != kW3 && fmt != kCB) {
    for (int ns : {2, 4}) {
      Plan q;
      if (make_plan(fmt, M, N, K, false, &q, ns) == cudaSuccess && q.ws_bytes > p.ws_bytes)
        p.ws_bytes = q.ws_bytes;
    }
  }
  // the outlier kernel (W4) may resolve to a different occupancy: cover both
  if (fmt == kW4 && N % 128 == 0) {
    Plan q;
    if (make_plan(fmt, M, N, K, true, &q) == cudaSuccess && q.ws_bytes > p.ws_bytes) return q.ws_bytes;
  }
  return p.ws_bytes;
}

extern "C" ql_status qlinear_plan(int fmt, int M, int N, int K, ql_plan* plan) {
  if (!plan) return QL_ERR_NULL;
  if (!gemv_fmt_ok(fmt)) return QL_ERR_UNSUPPORTED;
  if (!shape_ok(M, N, K)) return QL_ERR_SHAPE;
  Plan p;
  if (make_plan(fmt, M, N, K, false, &p) != cudaSuccess) return QL_ERR_CUDA;
  plan->ctas = p.C;
  plan->warps = p.NC;
  plan->tiles_per_warp = p.T;
  plan->units = p.U;
  plan->m_bucket = p.MT;
  plan->warps_per_unit = p.WPU;
  return QL_OK;
}

#define QL_UNIFORM_ENTRY(NAME, FMT)                                                              \
  extern "C" ql_status NAME(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,  \
                            const uint16_t* zeros, uint16_t* y, int M, int N, int K, int group,  \
                            void* workspace, size_t workspace_bytes, ql_stream_t stream) {       \
    const int ns = subgroups(group, K);                                                           \
    if (!ns) return QL_ERR_SHAPE;                                                                 \
    Call c{FMT, false, x, qweight, scales, zeros, nullptr, nullptr, nullptr, y, M, N, K,         \
           workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), ns};               \
    return run(c);                                                                                \
  }

QL_UNIFORM_ENTRY(qlinear_w4a16, kW4)
QL_UNIFORM_ENTRY(qlinear_w2a16, kW2)
QL_UNIFORM_ENTRY(qlinear_w8a16, kW8)

extern "C" ql_status qlinear_w3a16(const uint16_t* x, const uint32_t* qweight,
                                   const uint16_t* scales, const uint16_t* zeros, uint16_t* y,
                                   int M, int N, int K, int group, void* workspace,
                                   size_t workspace_bytes, ql_stream_t stream) {
  if (subgroups(group, K) != 1) return QL_ERR_SHAPE;  // group 128 or per-channel
  Call c{kW3, false, x, qweight, scales, zeros, nullptr, nullptr, nullptr, y, M, N, K,
         workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), 1};
  return run(c);
}

extern "C" ql_status qlinear_lut4(const uint16_t* x, const uint8_t* codes, const uint16_t* lut16,
                                  const float* absmax, uint16_t* y, int M, int N, int K, int block,
                                  void* workspace, size_t workspace_bytes, ql_stream_t stream) {
  if (block != kLutBlock) return QL_ERR_SHAPE;
  Call c{kLUT4, false, x, codes, lut16, absmax, nullptr, nullptr, nullptr, y, M, N, K,
         workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)};
  return run(c);
}

extern "C" ql_status qlinear_codebook_tc(const uint16_t* x, const uint8_t* codes,
                                         const uint16_t* scales, const uint16_t* codebook,
                                         uint16_t* y, int M, int N, int K, void* workspace,
                                         size_t workspace_bytes, ql_stream_t stream) {
  Call c{kCB, false, x, codes, scales, codebook, nullptr, nullptr, nullptr, y, M, N, K,
         workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)};
  return run(c);
}

extern "C" ql_status qlinear_w4a16_outlier(const uint16_t* x, const uint32_t* qweight,
                                           const uint16_t* scales, const uint16_t* zeros,
                                           const uint32_t* tile_offsets, const uint8_t* tile_rc,
                                           const uint16_t* tile_vals, uint16_t* y, int M, int N,
                                           int K, int group, void* workspace,
                                           size_t workspace_bytes, ql_stream_t stream) {
  if (group != kGroup) return QL_ERR_SHAPE;
  Call c{kW4, true, x, qweight, scales, zeros, tile_offsets, tile_rc, tile_vals, y, M, N, K,
         workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)};
  return run(c);
}

extern "C" ql_status qlinear_debug_unpack(int fmt, const void* packed, uint8_t* codes, int N,
                                          int K, ql_stream_t stream) {
  if (!fmt_ok(fmt)) return QL_ERR_UNSUPPORTED;
  if (!packed || !codes) return QL_ERR_NULL;
  if (!shape_ok(1, N, K)) return QL_ERR_SHAPE;
  if (!aligned(packed, 16)) return QL_ERR_ALIGN;
  return launch_debug<false>(fmt, packed, nullptr, nullptr, codes, nullptr, N, K,
                             reinterpret_cast<cudaStream_t>(stream));
}

extern "C" ql_status qlinear_debug_dequant(int fmt, const void* packed, const void* p0,
                                           const void* p1, float* w, int N, int K,
                                           ql_stream_t stream) {
  if (!fmt_ok(fmt)) return QL_ERR_UNSUPPORTED;
  if (!packed || !p0 || !p1 || !w) return QL_ERR_NULL;
  if (!shape_ok(1, N, K)) return QL_ERR_SHAPE;
  if (!aligned(packed, 16) || !aligned(w, 4)) return QL_ERR_ALIGN;
  if (fmt == kLUT4 ? !aligned(p1, 16) : (!aligned(p0, 4) || !aligned(p1, 4))) return QL_ERR_ALIGN;
  return launch_debug<true>(fmt, packed, p0, p1, nullptr, w, N, K,
                            reinterpret_cast<cudaStream_t>(stream));
}

extern "C" ql_status qlinear_debug_wait_test(uint32_t wait_limit, uint32_t producer_delay_us,
                                             uint32_t consumer_hold_us) {
  if (producer_delay_us > 0xFFFFu || consumer_hold_us > 0xFFFFu) return QL_ERR_SHAPE;
  g_wait_limit.store(wait_limit ? wait_limit : qlk::kSpinLimit, std::memory_order_relaxed);
  g_test_us.store(producer_delay_us | (consumer_hold_us << 16), std::memory_order_relaxed);
  return QL_OK;
}

extern "C" ql_status qlinear_read_error(void* workspace, uint32_t* flags, ql_stream_t stream) {
  if (!workspace || !flags) return QL_ERR_NULL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(flags, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return QL_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st) != cudaSuccess) return QL_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// W4A16 GEMV without a caller-provided workspace.
//
// Some callers cannot allocate device memory at all: plug-ins and embedded runtimes
// whose device memory is owned by a host application or a fixed pool they may not grow,
// and code that must not call cudaMalloc/cudaFree because those calls synchronize the
// device or are forbidden in its execution context.  For them this entry point keeps its
// split-K scratch (error word, arrival counters, partial sums) in a fixed array compiled
// into the library instead of a workspace argument.
//
// The array lives in every device's memory from the moment the library is loaded until
// the process exits.  In host code its name only stands in for it; the device address is
// looked up with cudaGetSymbolAddress, with the device current, on the first call made in
// a device's current context (so that first call should come before any stream capture),
// and looked up again when the context changes (after a device reset the module, and
// with it the array, may sit at another address).  All calls on a device share the array
// and it keeps the contents of the last call: the arrival counters are cleared on the
// call's stream before each launch, the error word stays set until
// qlinear_w4a16_noalloc_read_error reads it, and two calls whose device work overlaps
// (e.g. on two streams) race on it.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// The current context (cuCtxGetCurrent, looked up once through the runtime: no link
// against libcuda).  nullptr when it cannot be queried.
void* current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<Fn>(p);
  });
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

// Device address of g_noalloc_scratch on the current device: looked up once per device
// and context (again whenever no context could be queried, e.g. before the runtime made
// one current).
cudaError_t noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {nullptr};
  static void* ctx_of[kMaxDevices] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* ctx = current_context();
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev] || !ctx || ctx != ctx_of[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
    ctx_of[dev] = ctx;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" ql_status qlinear_w4a16_noalloc(const uint16_t* x, const uint32_t* qweight,
                                           const uint16_t* scales, const uint16_t* zeros,
                                           uint16_t* y, int M, int N, int K, int group,
                                           ql_stream_t stream) {
  if (group != kGroup) return QL_ERR_SHAPE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Call c{kW4, false, x, qweight, scales, zeros, nullptr, nullptr, nullptr, y, M, N, K,
         nullptr, kNoAllocScratchBytes, st};
  // every argument check before anything is enqueued on the stream
  const ql_status chk = check_call(c);
  if (chk != QL_OK) return chk;
  Plan p;
  if (make_plan(kW4, M, N, K, false, &p) != cudaSuccess) return QL_ERR_CUDA;
  if (p.ws_bytes > kNoAllocScratchBytes) return QL_ERR_WORKSPACE;  // beyond the fixed scratch
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return QL_ERR_CUDA;
  // the arrival counters must start at zero (the partial sums need not; the error word
  // keeps its flags until they are read)
  if (cudaMemsetAsync(static_cast<uint8_t*>(scratch) + p.counter_offset, 0,
                      p.partial_offset - p.counter_offset, st) != cudaSuccess)
    return QL_ERR_CUDA;
  c.ws = scratch;
  return run(c);
}

extern "C" ql_status qlinear_w4a16_noalloc_read_error(uint32_t* flags, ql_stream_t stream) {
  if (!flags) return QL_ERR_NULL;
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return QL_ERR_CUDA;
  return qlinear_read_error(scratch, flags, stream);
}
