// Stand-alone dequantization of the packed weights to fp16, and the prefill linear layer
// built on it: dequantize once into a dense fp16 [N][K] matrix, then one dense fp16 GEMM.
//
// This is the write-back form of the "Fast NF4 Dequantization Kernels for Large Language
// Model Inference" page (method section, technical framework: load the 4-bit codes,
// dequantize through a 64-byte shared-memory table, write FP16 back to global memory for
// the following matmul), applied to every packed format.  It serves the compute-bound
// regime that the QFactory page flags (assumption stress test and limitation 1: prefill
// and large batches), where a GEMV that re-reads the codes per 16-row slice loses to one
// dequantization plus a tensor-core GEMM.
//
// Output layout: W[n][k] (one row per output column, the weight layout of a linear layer),
// row stride K.  Each lane of a warp owns, per tensor-core step pair, eight consecutive k
// of one column (the packed fragment order), so it writes them as one 16-byte store; a
// warp store covers 8 rows x 64 contiguous bytes, whole 32-byte sectors.
//
// The dense GEMM is this library's tcgen05 kernel (prefill_tc.cu): y[M][N] = x[M][K] .
// W[N][K]^T, fp16 in and out, fp32 accumulation.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "dequant_frag.cuh"
#include "layout.h"
#include "qlinear.h"

// the tensor-core GEMM of prefill_tc.cu
ql_status qlinear_gemm_f16_tc(const uint16_t* x, const uint16_t* w, uint16_t* y, int M, int N,
                              int K, cudaStream_t st);

using namespace qlayout;

namespace {

bool aligned(const void* p, size_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

constexpr int kWarps = 8;  // chunks per CTA (one warp each)

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void stg128(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// W2 / W4 / W8: a lane's 64 weights of the chunk, fp16(s * (q - z)) (dequant_frag.cuh).
template <int FMT>
__device__ __forceinline__ void dequant_chunk_uniform(const uint32_t* wv, __half2 s_lo,
                                                      __half2 s_hi, float z_lo, float z_hi,
                                                      __half* out_lo, __half* out_hi) {
  __half2 zb[2][2];
  qdq::zero_bias<FMT>(z_lo, z_hi, zb);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 o = qdq::uniform_pair8<FMT>(wv, 2 * i, h, zb, h ? s_hi : s_lo);
      stg128((h ? out_hi : out_lo) + 32 * i, o.x, o.y, o.z, o.w);
    }
}

// LUT4: a lane's 64 weights of the chunk, fp16(fp32(lut[q]) * absmax).  am = the absmax of
// (rows gi, gi + 8) for k < 64 and (rows gi, gi + 8) for k >= 64.
__device__ __forceinline__ void dequant_chunk_lut4(const uint32_t* wv, const float* lut_s,
                                                   float4 am, __half* out_lo, __half* out_hi) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float a = (i >= 2) ? (h ? am.w : am.z) : (h ? am.y : am.x);
      const uint4 o = qdq::lut_pair8(wv, 2 * i, h, lut_s, a);
      stg128((h ? out_hi : out_lo) + 32 * i, o.x, o.y, o.z, o.w);
    }
}

// One warp per packed chunk (16 columns x 128 k), chunks in memory order so that
// consecutive warps read consecutive bytes.
template <int FMT>
__global__ void __launch_bounds__(32 * kWarps) dequant_fp16_kernel(
    const uint8_t* __restrict__ packed, const void* __restrict__ p0, const void* __restrict__ p1,
    __half* __restrict__ w, int N, int K, long long nchunks) {
  __shared__ float lut_s[16];
  if constexpr (FMT == kLUT4) {
    if (threadIdx.x < 16) lut_s[threadIdx.x] = __half2float(static_cast<const __half*>(p0)[threadIdx.x]);
    __syncthreads();
  }
  const int lane = threadIdx.x & 31;
  const long long ch = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (ch >= nchunks) return;
  const int G = K / kGroup, ntiles = N / kTileN;
  const long long per_block = (long long)G * kBlockTiles;
  const int b = (int)(ch / per_block);
  const int rem = (int)(ch - (long long)b * per_block);
  const int tb = tiles_in_block(b, ntiles);
  const int g = rem / tb, jj = rem - g * tb;
  const int j = b * kBlockTiles + jj;

  constexpr int KW = FMT == kW2 ? 4 : FMT == kW8 ? 16 : 8;
  uint32_t wv[KW];
  const uint8_t* src = packed + ch * chunk_bytes(FMT);
#pragma unroll
  for (int q = 0; q < KW / 4; ++q) {
    const uint4 v = ldg_stream(src + (size_t)(q * 32 + lane) * 16);
    wv[4 * q] = v.x; wv[4 * q + 1] = v.y; wv[4 * q + 2] = v.z; wv[4 * q + 3] = v.w;
  }
  const int gi = lane >> 2, t = lane & 3;
  __half* out_lo = w + (size_t)(j * kTileN + gi) * K + (size_t)g * kGroup + 8 * t;
  __half* out_hi = out_lo + (size_t)8 * K;
  if constexpr (FMT == kLUT4) {
    const float4 am = *reinterpret_cast<const float4*>(static_cast<const float*>(p1) + ch * 32 + gi * 4);
    dequant_chunk_lut4(wv, lut_s, am, out_lo, out_hi);
  } else {
    const __half2 s2 = *reinterpret_cast<const __half2*>(static_cast<const __half*>(p0) + ch * 16 + gi * 2);
    const __half2 z2 = *reinterpret_cast<const __half2*>(static_cast<const __half*>(p1) + ch * 16 + gi * 2);
    dequant_chunk_uniform<FMT>(wv, __low2half2(s2), __high2half2(s2), __low2float(z2),
                               __high2float(z2), out_lo, out_hi);
  }
}

bool fmt_ok(int fmt) { return fmt == kW2 || fmt == kW4 || fmt == kW8 || fmt == kLUT4; }

ql_status check_dequant(int fmt, const void* packed, const void* p0, const void* p1,
                        const void* w, int N, int K) {
  if (!fmt_ok(fmt)) return QL_ERR_UNSUPPORTED;
  if (!packed || !p0 || !p1 || !w) return QL_ERR_NULL;
  if (N <= 0 || K <= 0 || N % kTileN || K % kGroup) return QL_ERR_SHAPE;
  if (!aligned(packed, 16) || !aligned(w, 16)) return QL_ERR_ALIGN;
  if (fmt == kLUT4 ? (!aligned(p0, 2) || !aligned(p1, 16)) : (!aligned(p0, 4) || !aligned(p1, 4)))
    return QL_ERR_ALIGN;
  return QL_OK;
}

ql_status launch_dequant(int fmt, const void* packed, const void* p0, const void* p1, void* w,
                         int N, int K, cudaStream_t st) {
  const long long nchunks = (long long)(N / kTileN) * (K / kGroup);
  const unsigned grid = (unsigned)((nchunks + kWarps - 1) / kWarps);
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  __half* out = static_cast<__half*>(w);
  switch (fmt) {
    case kW2: dequant_fp16_kernel<kW2><<<grid, 32 * kWarps, 0, st>>>(pk, p0, p1, out, N, K, nchunks); break;
    case kW4: dequant_fp16_kernel<kW4><<<grid, 32 * kWarps, 0, st>>>(pk, p0, p1, out, N, K, nchunks); break;
    case kW8: dequant_fp16_kernel<kW8><<<grid, 32 * kWarps, 0, st>>>(pk, p0, p1, out, N, K, nchunks); break;
    default: dequant_fp16_kernel<kLUT4><<<grid, 32 * kWarps, 0, st>>>(pk, p0, p1, out, N, K, nchunks); break;
  }
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

}  // namespace

// ---------------------------------------------------------------------------
// exported entry points

extern "C" ql_status qlinear_dequant_fp16(int fmt, const void* packed, const void* p0,
                                          const void* p1, uint16_t* w, int N, int K,
                                          ql_stream_t stream) {
  const ql_status st = check_dequant(fmt, packed, p0, p1, w, N, K);
  if (st != QL_OK) return st;
  return launch_dequant(fmt, packed, p0, p1, w, N, K, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" ql_status qlinear_prefill(int fmt, const uint16_t* x, const void* packed,
                                     const void* p0, const void* p1, uint16_t* w_fp16, uint16_t* y,
                                     int M, int N, int K, ql_stream_t stream) {
  if (!fmt_ok(fmt)) return QL_ERR_UNSUPPORTED;
  if (!x || !y) return QL_ERR_NULL;
  ql_status st = check_dequant(fmt, packed, p0, p1, w_fp16, N, K);
  if (st != QL_OK) return st;
  if (M <= 0) return QL_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(y, 2)) return QL_ERR_ALIGN;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  st = launch_dequant(fmt, packed, p0, p1, w_fp16, N, K, cs);
  if (st != QL_OK) return st;
  return qlinear_gemm_f16_tc(x, w_fp16, y, M, N, K, cs);
}
