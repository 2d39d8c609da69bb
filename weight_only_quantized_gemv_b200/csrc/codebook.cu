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
// Work split: K is cut into R ranges of SL 4-slices (64 at M = 1, 32 at M = 2, 16 at
// M = 3, 4: the Psumbook of a range, SL x 256 entries x the rows padded to 1, 2 or 4, is
// 64 KB), the tiles into P partitions; CTA (r, p) builds range r's Psumbook once and
// streams the codes of its tiles, each warp loading the next tile's codes before it works
// through the current one.  Each warp leaves one fp32 partial per (row, column) and range
// for each of its tiles, publishes them once at its end (one fence, one arrival per tile),
// and the warp that arrives last at a tile sums the R partials in range order
// (deterministic) and stores fp16.  A group's scale multiplies the sum of each 16 lookups of that group.
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

// Rows of x padded to a vector width: the Psumbook keeps the MP rows of one (slice, code)
// entry side by side, so one 4-, 8- or 16-byte lookup serves every row.
template <int MR>
__host__ __device__ constexpr int cb_mp() { return MR == 1 ? 1 : MR == 2 ? 2 : 4; }

// Slices (4-vectors along K) per K range: the Psumbook of a range is SL x 256 x MP fp32 =
// 64 KB for every M, three CTAs per SM.
template <int MR>
__host__ __device__ constexpr int cb_sl() { return MR == 1 ? 64 : MR == 2 ? 32 : 16; }

template <int MR>
__host__ __device__ constexpr int cb_smem_bytes() {
  return cb_sl<MR>() * kCbEntries * cb_mp<MR>() * 4 + MR * cb_sl<MR>() * kCbVec * 4;
}

template <int MP>
struct CbVecT;
template <> struct CbVecT<1> { using T = float; };
template <> struct CbVecT<2> { using T = float2; };
template <> struct CbVecT<4> { using T = float4; };

__device__ __forceinline__ void cb_add(float (&a)[4], float v) { a[0] += v; }
__device__ __forceinline__ void cb_add(float (&a)[4], float2 v) { a[0] += v.x; a[1] += v.y; }
__device__ __forceinline__ void cb_add(float (&a)[4], float4 v) {
  a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
}

template <int MR>
__global__ void __launch_bounds__(kCbThreads, 3) codebook_psum_kernel(const CbParams P) {
  constexpr int MP = cb_mp<MR>(), SL = cb_sl<MR>(), NQ = SL / 16;
  using VecT = typename CbVecT<MP>::T;
  extern __shared__ __align__(16) float cb_smem[];
  float* psum = cb_smem;                               // [SL][256][MP]
  float* xs = cb_smem + SL * kCbEntries * MP;          // [MR][SL * 4]
  const int r = blockIdx.x % P.R, part = blockIdx.x / P.R;
  const int J = P.K / kCbVec;                          // slices in K
  const int j0 = r * SL;
  const int nsl = min(SL, J - j0);                     // a multiple of 16 (K % 128 == 0)
  const int tid = threadIdx.x;

  // -- Psumbook of slices j0 .. j0 + nsl - 1 ---------------------------------------------
  for (int i = tid; i < MR * nsl * kCbVec; i += kCbThreads) {
    const int m = i / (nsl * kCbVec), e = i - m * nsl * kCbVec;
    xs[m * SL * kCbVec + e] = __half2float(P.x[(size_t)m * P.K + (size_t)j0 * kCbVec + e]);
  }
  __syncthreads();
  {
    const uint2 cw = reinterpret_cast<const uint2*>(P.codebook)[tid];  // centroid tid
    const float2 c01 = __half22float2(*reinterpret_cast<const __half2*>(&cw.x));
    const float2 c23 = __half22float2(*reinterpret_cast<const __half2*>(&cw.y));
#pragma unroll 4
    for (int j = 0; j < nsl; ++j) {
      float pv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        const float4 xv = *reinterpret_cast<const float4*>(xs + m * SL * kCbVec + 4 * j);
        pv[m] = fmaf(c23.y, xv.w, fmaf(c23.x, xv.z, fmaf(c01.y, xv.y, c01.x * xv.x)));
      }
      float* dst = psum + ((size_t)j * kCbEntries + tid) * MP;
      if constexpr (MP == 1) dst[0] = pv[0];
      else if constexpr (MP == 2) *reinterpret_cast<float2*>(dst) = make_float2(pv[0], pv[1]);
      else *reinterpret_cast<float4*>(dst) = make_float4(pv[0], pv[1], pv[2], pv[3]);
    }
  }
  __syncthreads();

  // -- stream the tiles: one lookup and one add per code, codes prefetched a tile ahead ---
  const int warp = tid >> 5, lane = tid & 31;
  const int stride = P.P * (kCbThreads / 32);
  const int nq = nsl / 16;
  // quad qi of the range: slices j0 + 16 qi .. + 15, i.e. half (j0 / 16 + qi) % 2 of group
  // (j0 / 16 + qi) / 2
  auto load = [&](int T, uint4 (&cq)[NQ], float (&sc)[NQ]) {
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
      if (qi < nq) {
        const int b16 = j0 / 16 + qi;
        const size_t ch = (size_t)T * P.G + (b16 >> 1);
        cq[qi] = ldg_stream(P.codes + ch * (kCbTile * kCbSlices) + (size_t)((b16 & 1) * 32 + lane) * 16);
        sc[qi] = __half2float(P.scales[ch * kCbTile + lane]);
      }
    }
  };
  int T = part * (kCbThreads / 32) + warp;
  uint4 cq[NQ];
  float sc[NQ];
  if (T < P.ntiles) load(T, cq, sc);
  while (T < P.ntiles) {
    const int Tn = T + stride;
    uint4 nq4[NQ];
    float nsc[NQ];
    if (Tn < P.ntiles) load(Tn, nq4, nsc);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
      if (qi >= nq) break;
      const uint32_t w[4] = {cq[qi].x, cq[qi].y, cq[qi].z, cq[qi].w};
      const VecT* tab = reinterpret_cast<const VecT*>(psum) + qi * 16 * kCbEntries;
      float s4[4][4] = {};
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t code = __byte_perm(w[j >> 2], 0u, 0x4440u | (uint32_t)(j & 3));
        cb_add(s4[j & 3], tab[j * kCbEntries + code]);
      }
#pragma unroll
      for (int m = 0; m < MR; ++m)
        acc[m] = fmaf(sc[qi], (s4[0][m] + s4[1][m]) + (s4[2][m] + s4[3][m]), acc[m]);
    }
    const int n = T * kCbTile + lane;
    if (P.R == 1) {
#pragma unroll
      for (int m = 0; m < MR; ++m) P.y[(size_t)m * P.N + n] = __float2half_rn(acc[m]);
    } else {
#pragma unroll
      for (int m = 0; m < MR; ++m) P.partials[((size_t)r * MR + m) * P.N + n] = acc[m];
    }
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
      cq[qi] = nq4[qi];
      sc[qi] = nsc[qi];
    }
    T = Tn;
  }
  if (P.R == 1) return;

  // -- publish this warp's partials once, then finish the tiles it reached last ---------
  // (a fence per tile would wait for the prefetched codes of the next tile every time)
  const int T0 = part * (kCbThreads / 32) + warp;
  const int cnt = T0 < P.ntiles ? (P.ntiles - 1 - T0) / stride + 1 : 0;
  __threadfence();
  __syncwarp();
  for (int b = 0; b < cnt; b += 32) {
    bool last = false;
    if (b + lane < cnt) {
      uint32_t old;
      asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old)
                   : "l"(P.counters + T0 + (b + lane) * stride) : "memory");
      last = old == (uint32_t)(P.R - 1);
    }
    uint32_t mask = __ballot_sync(0xffffffffu, last);
    if (mask) __threadfence();
    while (mask) {  // tiles whose every range has arrived: sum the R partials in range order
      const int i = __ffs(mask) - 1;
      mask &= mask - 1;
      const int Tl = T0 + (b + i) * stride;
      const int nl = Tl * kCbTile + lane;
      // loads issued eight ranges at a time (independent, so their latencies overlap),
      // added in range order
      float t[MR];
#pragma unroll
      for (int m = 0; m < MR; ++m) t[m] = 0.f;
      const float* pp = P.partials + nl;
      const size_t rs = (size_t)MR * P.N;
      int rr = 0;
      for (; rr + 8 <= P.R; rr += 8) {
        float v[8][MR];
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int m = 0; m < MR; ++m) v[u][m] = __ldcg(pp + (size_t)(rr + u) * rs + (size_t)m * P.N);
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int m = 0; m < MR; ++m) t[m] += v[u][m];
      }
      for (; rr < P.R; ++rr)
#pragma unroll
        for (int m = 0; m < MR; ++m) t[m] += __ldcg(pp + (size_t)rr * rs + (size_t)m * P.N);
#pragma unroll
      for (int m = 0; m < MR; ++m) P.y[(size_t)m * P.N + nl] = __float2half_rn(t[m]);
      if (lane == 0) P.counters[Tl] = 0u;  // ready for the next call
    }
  }
}

struct CbKernel {
  const void* fn;
  int smem, SL;
};

template <int MR>
CbKernel cb_kernel() {
  return CbKernel{reinterpret_cast<const void*>(codebook_psum_kernel<MR>), cb_smem_bytes<MR>(),
                  cb_sl<MR>()};
}

CbKernel select_cb(int M) {
  switch (M) {
    case 1: return cb_kernel<1>();
    case 2: return cb_kernel<2>();
    case 3: return cb_kernel<3>();
    default: return cb_kernel<4>();
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
  const int J = K / kCbVec;
  p->R = (J + p->k.SL - 1) / p->k.SL;
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
