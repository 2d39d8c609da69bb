// Codebook GEMV with a Psumbook (CodeGEMM page, method: overall framework and key
// designs one, two and four), configuration m1v4g128: one codebook C of 256 fp16
// 4-vectors, one 8-bit code per 4 consecutive k of a column (2 bits per weight), one
// fp16 normalization scale per 128 k of a column:
//
//   w[k][n] = s[k / 128][n] * C[code[k / 4][n]][k % 4]
//   y[m][n] = sum_g s[g][n] * sum_{j in g} P[m][j][code[j][n]],   P[m][j][i] = C[i] . x[m][4j .. 4j+3]
//
// Instead of rebuilding weights, each CTA builds the Psumbook of its K range in shared
// memory (every 4-slice of x against all 256 centroids, fp32) and then replaces each
// 4-weight dot product by one table lookup and one add.
//
// Packed layout (qlinear_pack_codebook): 32-column tiles T (column n = 32 T + lane) by
// 128-k groups g; chunk (T, g) = T * G + g holds 1024 bytes, lane l's 32 codes (the
// group's 4-vectors j = 0..31 in order) as two 16-byte quads at byte ((j / 16) * 32 + l) * 16
// + j % 16, so one warp reads a chunk with two coalesced 512-byte loads.  Scales follow the
// chunk order: fp16 [T][g][lane].
//
// Work split: the groups are cut into R ranges of GC groups (the Psumbook of a range fits
// in shared memory), the tiles into P partitions; CTA (r, p) builds range r's Psumbook
// once and streams the chunks of its tiles.  Each warp leaves one fp32 partial per (row,
// column) and range; the last warp to arrive at a tile sums the R partials in range order
// (deterministic) and stores fp16.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <unordered_map>

#include "qlinear.h"

namespace {

constexpr int kCbThreads = 256;
constexpr int kCbTile = 32;      // columns per tile (one per lane)
constexpr int kCbGroup = 128;    // normalization group along K
constexpr int kCbVec = 4;        // weights per code
constexpr int kCbSlices = kCbGroup / kCbVec;  // 32 codes per column per group
constexpr int kCbEntries = 256;

bool aligned(const void* p, size_t a) { return ((uintptr_t)p & (a - 1)) == 0; }
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct CbParams {
  const __half* x;
  const uint8_t* codes;
  const __half* scales;
  const __half* codebook;
  __half* y;
  float* partials;     // [R][M][N]
  uint32_t* counters;  // [ntiles]
  int M, N, K, G, R, P, ntiles;
};

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <int MR, int GC>
constexpr int cb_smem_bytes() {
  return MR * GC * kCbSlices * kCbEntries * 4 + MR * GC * kCbGroup * 4;
}

template <int MR, int GC>
__global__ void __launch_bounds__(kCbThreads, (MR * GC <= 2) ? 3 : 1)
    codebook_psum_kernel(const CbParams P) {
  extern __shared__ __align__(16) float cb_smem[];
  float* psum = cb_smem;                                         // [MR][GC][32][256]
  float* xs = cb_smem + MR * GC * kCbSlices * kCbEntries;        // [MR][GC * 128]
  const int r = blockIdx.x % P.R, part = blockIdx.x / P.R;
  const int g0 = r * GC;
  const int gc = min(GC, P.G - g0);
  const int tid = threadIdx.x;

  // -- Psumbook of groups g0 .. g0 + gc - 1 -------------------------------------------
  for (int i = tid; i < MR * gc * kCbGroup; i += kCbThreads) {
    const int m = i / (gc * kCbGroup), e = i - m * gc * kCbGroup;
    xs[m * GC * kCbGroup + e] = __half2float(P.x[(size_t)m * P.K + (size_t)g0 * kCbGroup + e]);
  }
  __syncthreads();
  {
    const uint2 cw = reinterpret_cast<const uint2*>(P.codebook)[tid];  // centroid tid
    const float2 c01 = __half22float2(*reinterpret_cast<const __half2*>(&cw.x));
    const float2 c23 = __half22float2(*reinterpret_cast<const __half2*>(&cw.y));
#pragma unroll
    for (int m = 0; m < MR; ++m)
      for (int gg = 0; gg < gc; ++gg)
#pragma unroll 8
        for (int j = 0; j < kCbSlices; ++j) {
          const float4 xv = *reinterpret_cast<const float4*>(xs + m * GC * kCbGroup + gg * kCbGroup + 4 * j);
          const float p = fmaf(c23.y, xv.w, fmaf(c23.x, xv.z, fmaf(c01.y, xv.y, c01.x * xv.x)));
          psum[((m * GC + gg) * kCbSlices + j) * kCbEntries + tid] = p;
        }
  }
  __syncthreads();

  // -- stream the tiles: one lookup and one add per code ---------------------------------
  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t psum_s = (uint32_t)__cvta_generic_to_shared(psum);
  for (int T = part * (kCbThreads / 32) + warp; T < P.ntiles; T += P.P * (kCbThreads / 32)) {
    float acc[MR];
#pragma unroll
    for (int m = 0; m < MR; ++m) acc[m] = 0.f;
    uint4 cq[GC][2];
    float sc[GC];
#pragma unroll
    for (int gg = 0; gg < GC; ++gg) {
      if (gg < gc) {
        const size_t ch = (size_t)T * P.G + g0 + gg;
        const uint8_t* src = P.codes + ch * (kCbTile * kCbSlices);
        cq[gg][0] = ldg_stream(src + (size_t)lane * 16);
        cq[gg][1] = ldg_stream(src + (size_t)(32 + lane) * 16);
        sc[gg] = __half2float(P.scales[ch * kCbTile + lane]);
      }
    }
#pragma unroll
    for (int gg = 0; gg < GC; ++gg) {
      if (gg >= gc) break;
      const uint32_t w[8] = {cq[gg][0].x, cq[gg][0].y, cq[gg][0].z, cq[gg][0].w,
                             cq[gg][1].x, cq[gg][1].y, cq[gg][1].z, cq[gg][1].w};
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t base = psum_s + (uint32_t)((m * GC + gg) * kCbSlices * kCbEntries * 4);
#pragma unroll
        for (int j = 0; j < kCbSlices; ++j) {
          const uint32_t code = (w[j >> 2] >> (8 * (j & 3))) & 0xFFu;
          float v;
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v)
                       : "r"(base + (uint32_t)(j * kCbEntries * 4) + code * 4u));
          s4[j & 3] += v;
        }
        acc[m] = fmaf(sc[gg], (s4[0] + s4[1]) + (s4[2] + s4[3]), acc[m]);
      }
    }
    const int n = T * kCbTile + lane;
    if (P.R == 1) {
#pragma unroll
      for (int m = 0; m < MR; ++m) P.y[(size_t)m * P.N + n] = __float2half_rn(acc[m]);
      continue;
    }
#pragma unroll
    for (int m = 0; m < MR; ++m) P.partials[((size_t)r * MR + m) * P.N + n] = acc[m];
    __threadfence();
    __syncwarp();
    uint32_t old = 0;
    if (lane == 0) {
      asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(P.counters + T) : "memory");
    }
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old == (uint32_t)(P.R - 1)) {  // last range to arrive: sum all R in range order
      __threadfence();
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        float t = 0.f;
        for (int rr = 0; rr < P.R; ++rr) t += __ldcg(P.partials + ((size_t)rr * MR + m) * P.N + n);
        P.y[(size_t)m * P.N + n] = __float2half_rn(t);
      }
      if (lane == 0) P.counters[T] = 0u;  // ready for the next call
    }
  }
}

struct CbKernel {
  const void* fn;
  int smem, GC;
};

template <int MR, int GC>
CbKernel cb_kernel() {
  return CbKernel{reinterpret_cast<const void*>(codebook_psum_kernel<MR, GC>), cb_smem_bytes<MR, GC>(),
                  GC};
}

CbKernel select_cb(int M) {
  switch (M) {
    case 1: return cb_kernel<1, 2>();
    case 2: return cb_kernel<2, 1>();
    case 3: return cb_kernel<3, 1>();
    default: return cb_kernel<4, 1>();
  }
}

struct CbPlan {
  CbKernel k;
  int R, P, ntiles, G;
  size_t partial_offset, ws_bytes;
};

cudaError_t cb_plan(int M, int N, int K, CbPlan* p) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  p->k = select_cb(M);
  static std::mutex mu;
  static std::unordered_map<uint64_t, int> occ_cache;
  int occ = 1;
  {
    std::lock_guard<std::mutex> lk(mu);
    const uint64_t key = ((uint64_t)(uintptr_t)p->k.fn << 8) ^ (uint64_t)dev;
    auto it = occ_cache.find(key);
    if (it != occ_cache.end()) {
      occ = it->second;
    } else {
      e = cudaFuncSetAttribute(p->k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, p->k.smem);
      if (e != cudaSuccess) return e;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, p->k.fn, kCbThreads, p->k.smem);
      if (e != cudaSuccess) return e;
      if (occ < 1) occ = 1;
      occ_cache[key] = occ;
    }
  }
  p->G = K / kCbGroup;
  p->ntiles = N / kCbTile;
  p->R = (p->G + p->k.GC - 1) / p->k.GC;
  const long long slots = (long long)sms * occ;
  const long long tile_rows = (p->ntiles + kCbThreads / 32 - 1) / (kCbThreads / 32);
  long long parts = slots / p->R;
  if (parts < 1) parts = 1;
  if (parts > tile_rows) parts = tile_rows;
  p->P = (int)parts;
  p->partial_offset = align_up((size_t)p->ntiles * sizeof(uint32_t), 256);
  p->ws_bytes = p->partial_offset + (p->R > 1 ? (size_t)p->R * M * N * sizeof(float) : 0);
  if ((long long)p->R * p->P >= (1LL << 31)) return cudaErrorInvalidValue;
  return cudaSuccess;
}

bool cb_shape_ok(int M, int N, int K) {
  return M >= 1 && M <= 4 && N > 0 && K > 0 && N % kCbTile == 0 && K % kCbGroup == 0;
}

}  // namespace

// ---------------------------------------------------------------------------
// host packers

extern "C" ql_status qlinear_pack_codebook(const uint8_t* codes, uint8_t* packed, int N, int K) {
  if (!codes || !packed) return QL_ERR_NULL;
  if (N <= 0 || K <= 0 || N % kCbTile || K % kCbGroup) return QL_ERR_SHAPE;
  const int G = K / kCbGroup, ntiles = N / kCbTile;
  for (int T = 0; T < ntiles; ++T)
    for (int g = 0; g < G; ++g) {
      uint8_t* ch = packed + ((size_t)T * G + g) * (kCbTile * kCbSlices);
      for (int l = 0; l < kCbTile; ++l)
        for (int j = 0; j < kCbSlices; ++j)
          ch[((j / 16) * 32 + l) * 16 + j % 16] =
              codes[(size_t)(g * kCbSlices + j) * N + (size_t)T * kCbTile + l];
    }
  return QL_OK;
}

extern "C" ql_status qlinear_pack_codebook_scales(const uint16_t* scales, uint16_t* packed, int N,
                                                  int K) {
  if (!scales || !packed) return QL_ERR_NULL;
  if (N <= 0 || K <= 0 || N % kCbTile || K % kCbGroup) return QL_ERR_SHAPE;
  const int G = K / kCbGroup, ntiles = N / kCbTile;
  for (int T = 0; T < ntiles; ++T)
    for (int g = 0; g < G; ++g)
      for (int l = 0; l < kCbTile; ++l)
        packed[((size_t)T * G + g) * kCbTile + l] = scales[(size_t)g * N + (size_t)T * kCbTile + l];
  return QL_OK;
}

// ---------------------------------------------------------------------------
// GEMV

extern "C" size_t qlinear_codebook_workspace_bytes(int M, int N, int K) {
  if (!cb_shape_ok(M, N, K)) return 0;
  CbPlan p;
  if (cb_plan(M, N, K, &p) != cudaSuccess) return 0;
  return p.ws_bytes;
}

extern "C" ql_status qlinear_codebook(const uint16_t* x, const uint8_t* codes,
                                      const uint16_t* scales, const uint16_t* codebook,
                                      uint16_t* y, int M, int N, int K, void* workspace,
                                      size_t workspace_bytes, ql_stream_t stream) {
  if (!x || !codes || !scales || !codebook || !y) return QL_ERR_NULL;
  if (!cb_shape_ok(M, N, K)) return QL_ERR_SHAPE;
  if (!aligned(x, 2) || !aligned(codes, 16) || !aligned(scales, 2) || !aligned(codebook, 8) ||
      !aligned(y, 2))
    return QL_ERR_ALIGN;
  CbPlan p;
  if (cb_plan(M, N, K, &p) != cudaSuccess) return QL_ERR_CUDA;
  if (p.R > 1) {
    if (!workspace || workspace_bytes < p.ws_bytes) return QL_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return QL_ERR_ALIGN;
  }
  CbParams P;
  P.x = reinterpret_cast<const __half*>(x);
  P.codes = codes;
  P.scales = reinterpret_cast<const __half*>(scales);
  P.codebook = reinterpret_cast<const __half*>(codebook);
  P.y = reinterpret_cast<__half*>(y);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  P.counters = reinterpret_cast<uint32_t*>(ws);
  P.partials = p.R > 1 ? reinterpret_cast<float*>(ws + p.partial_offset) : nullptr;
  P.M = M;
  P.N = N;
  P.K = K;
  P.G = p.G;
  P.R = p.R;
  P.P = p.P;
  P.ntiles = p.ntiles;
  void* args[1] = {&P};
  const dim3 grid((unsigned)(p.R * p.P)), block(kCbThreads);
  if (cudaLaunchKernel(p.k.fn, grid, block, args, (size_t)p.k.smem,
                       reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return QL_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}
