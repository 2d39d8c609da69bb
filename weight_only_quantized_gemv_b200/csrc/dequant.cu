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
// The dense GEMM is cuBLAS (opened at run time with dlopen, so loading this library needs
// neither cuBLAS nor a GPU): y[M][N] = x[M][K] . W[N][K]^T, fp16 in and out, fp32
// accumulation.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cublas_v2.h>  // types and prototypes only; the library is opened with dlopen
#include <dlfcn.h>

#include <mutex>
#include <unordered_map>

#include "layout.h"
#include "qlinear.h"

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

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}

// Bit offset (inside each 16-bit half of fragment register r of step s) of the code field
// that the AND masks below leave in place.
template <int FMT>
__device__ __forceinline__ constexpr int field_shift(int s, int r) {
  return FMT == kW4 ? ((r & 1) ? 4 : 0) : FMT == kW2 ? 4 * (s & 1) + ((r & 1) ? 2 : 0) : 0;
}

// The code fields of fragment register r of step s, each in its own 16-bit half (low half =
// the smaller k), at the bit offsets field_shift() gives.
template <int FMT>
__device__ __forceinline__ uint32_t code_fields(const uint32_t* w, int s, int r) {
  if constexpr (FMT == kW4) {
    const uint32_t v = (r >> 1) ? (w[s] >> 8) : w[s];
    return v & ((r & 1) ? 0x00F000F0u : 0x000F000Fu);
  } else if constexpr (FMT == kW2) {
    const uint32_t v = (r >> 1) ? (w[s >> 1] >> 8) : w[s >> 1];
    const uint32_t m = (r & 1) ? ((s & 1) ? 0x00C000C0u : 0x000C000Cu)
                               : ((s & 1) ? 0x00300030u : 0x00030003u);
    return v & m;
  } else {  // W8: words 2s (rows gi) and 2s + 1 (rows gi + 8)
    const uint32_t v = (r >> 1) ? (w[2 * s + (r & 1)] >> 8) : w[2 * s + (r & 1)];
    return v & 0x00FF00FFu;
  }
}

// fp16 bit pattern of 2^(10 - sh): its last mantissa bit weighs 2^-sh, so OR-ing a code
// field that sits at bit offset sh into the mantissa gives exactly 2^(10 - sh) + q.
__device__ __forceinline__ constexpr uint32_t magic_half(int sh) {
  return (uint32_t)(25 - sh) << 10;
}

// W2 / W4 / W8: w = fp16(s * (q - z)).  (2^(10-sh) + q) - (2^(10-sh) + z) = q - z is exact
// in fp16 (|q - z| <= 255 < 2^11), and the fp16 product rounds the exact s (q - z) once.
template <int FMT>
__device__ __forceinline__ void dequant_chunk_uniform(const uint32_t* wv, __half2 s_lo,
                                                      __half2 s_hi, float z_lo, float z_hi,
                                                      __half* out_lo, __half* out_hi) {
  // z + 2^(10 - sh) per (step parity, row half): exact small integers / dyadics in fp16
  __half2 zb[2][2];
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int sh = field_shift<FMT>(p, h);
      zb[p][h] = __float2half2_rn((float)(1 << (10 - sh)) + (h ? z_hi : z_lo));
    }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t o[4];
#pragma unroll
      for (int ss = 0; ss < 2; ++ss)
#pragma unroll
        for (int dkp = 0; dkp < 2; ++dkp) {
          const int s = 2 * i + ss, r = h + 2 * dkp;
          const uint32_t f = code_fields<FMT>(wv, s, r) | (magic_half(field_shift<FMT>(s, r)) * 0x10001u);
          const __half2 d = __hsub2(u32_as_h2(f), zb[s & 1][h]);
          o[2 * ss + dkp] = h2_as_u32(__hmul2(d, h ? s_hi : s_lo));
        }
      stg128((h ? out_hi : out_lo) + 32 * i, o[0], o[1], o[2], o[3]);
    }
}

// LUT4: w = fp16(fp32(lut[q]) * absmax) with the product rounded to fp32 first.  Byte r of
// word s holds the two codes of fragment register r (low nibble = the smaller k).
__device__ __forceinline__ void dequant_chunk_lut4(const uint32_t* wv, const float* lut_s,
                                                   float4 am, __half* out_lo, __half* out_hi) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t o[4];
#pragma unroll
      for (int ss = 0; ss < 2; ++ss)
#pragma unroll
        for (int dkp = 0; dkp < 2; ++dkp) {
          const int s = 2 * i + ss, r = h + 2 * dkp;
          // absmax block: k in the group < 64 for steps 0..3; (x, y) = rows (gi, gi + 8)
          const float a = (s >= 4) ? (h ? am.w : am.z) : (h ? am.y : am.x);
          const uint32_t byte = (wv[s] >> (8 * r)) & 0xFFu;
          const float lo = __fmul_rn(lut_s[byte & 0xFu], a);
          const float hi = __fmul_rn(lut_s[byte >> 4], a);
          o[2 * ss + dkp] = h2_as_u32(__floats2half2_rn(lo, hi));
        }
      stg128((h ? out_hi : out_lo) + 32 * i, o[0], o[1], o[2], o[3]);
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

// ---------------------------------------------------------------------------
// cuBLAS, opened at run time

// the C symbol cublasGemmEx (C++ also sees an inline overload taking cudaDataType)
using GemmEx = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int,
                                  int, const void*, const void*, cudaDataType, int, const void*,
                                  cudaDataType, int, const void*, void*, cudaDataType, int,
                                  cublasComputeType_t, cublasGemmAlgo_t);

struct Blas {
  decltype(&cublasCreate_v2) create = nullptr;
  decltype(&cublasSetStream_v2) set_stream = nullptr;
  GemmEx gemm = nullptr;
  bool ok = false;
};

const Blas& blas() {
  static Blas b;
  static std::once_flag once;
  std::call_once(once, [] {
    void* h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_GLOBAL);
    if (!h) h = dlopen("libcublas.so", RTLD_NOW | RTLD_GLOBAL);
    if (!h) return;
    b.create = reinterpret_cast<decltype(&cublasCreate_v2)>(dlsym(h, "cublasCreate_v2"));
    b.set_stream = reinterpret_cast<decltype(&cublasSetStream_v2)>(dlsym(h, "cublasSetStream_v2"));
    b.gemm = reinterpret_cast<GemmEx>(dlsym(h, "cublasGemmEx"));
    b.ok = b.create && b.set_stream && b.gemm;
  });
  return b;
}

// One handle per (thread, device), created on first use and kept for the process.
cublasHandle_t blas_handle(const Blas& b) {
  thread_local std::unordered_map<int, cublasHandle_t> handles;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  auto it = handles.find(dev);
  if (it != handles.end()) return it->second;
  cublasHandle_t h = nullptr;
  if (b.create(&h) != CUBLAS_STATUS_SUCCESS) return nullptr;
  handles.emplace(dev, h);
  return h;
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
  if (!aligned(x, 2) || !aligned(y, 2)) return QL_ERR_ALIGN;
  const Blas& b = blas();
  if (!b.ok) return QL_ERR_LIBRARY;
  cublasHandle_t h = blas_handle(b);
  if (!h) return QL_ERR_LIBRARY;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  st = launch_dequant(fmt, packed, p0, p1, w_fp16, N, K, cs);
  if (st != QL_OK) return st;
  if (b.set_stream(h, cs) != CUBLAS_STATUS_SUCCESS) return QL_ERR_LIBRARY;
  const float one = 1.0f, zero = 0.0f;
  // column-major view: y^T (N x M, ld N) = W^T (op T of the K x N view of W[N][K], ld K)
  //                                        . x^T (K x M view of x[M][K], ld K)
  const cublasStatus_t cs2 = b.gemm(h, CUBLAS_OP_T, CUBLAS_OP_N, N, M, K, &one, w_fp16, CUDA_R_16F,
                                    K, x, CUDA_R_16F, K, &zero, y, CUDA_R_16F, N,
                                    CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
  return cs2 == CUBLAS_STATUS_SUCCESS ? QL_OK : QL_ERR_CUDA;
}
