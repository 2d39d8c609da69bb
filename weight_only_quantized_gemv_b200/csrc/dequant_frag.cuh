// Decoding of the packed weight layout into fp16 weights, eight consecutive k of one column
// at a time (one 16-byte value): shared by the stand-alone dequantization kernel, which
// writes them to global memory, and the prefill GEMM, which writes them into the shared-
// memory operand of its tensor-core MMAs.
//
// In a packed 16 x 128 chunk, lane (gi = lane / 4, t = lane % 4) holds the A fragments of
// the eight tensor-core steps s for columns gi and gi + 8.  Steps 2i and 2i + 1 together
// cover k = 32 i + 8 t + 0..7 of both columns (layout.h), so a lane turns each step pair
// into two 16-byte values: one for column gi (h = 0), one for column gi + 8 (h = 1).
//
// Word arrays passed to these helpers may hold the chunk's words from any even step on:
// the functions read step s through its word index and its parity only, so a caller that
// loaded only the words of steps 4 .. 7 passes them as steps 0 .. 3.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "layout.h"

namespace qdq {

using namespace qlayout;

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Bit offset (inside each 16-bit half of fragment register r of step s) of the code field
// that the AND masks of code_fields() leave in place.
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
__device__ __forceinline__ constexpr uint32_t magic_half(int sh) { return (uint32_t)(25 - sh) << 10; }

// z + 2^(10 - sh) per (step parity, row half): exact small integers / dyadics in fp16.
template <int FMT>
__device__ __forceinline__ void zero_bias(float z_lo, float z_hi, __half2 (&zb)[2][2]) {
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int h = 0; h < 2; ++h)
      zb[p][h] = __float2half2_rn((float)(1 << (10 - field_shift<FMT>(p, h))) + (h ? z_hi : z_lo));
}

// W2 / W4 / W8: the eight fp16 weights fp16(s * (q - z)) of steps s0, s0 + 1 (s0 even) for
// row half h.  (2^(10-sh) + q) - (2^(10-sh) + z) = q - z is exact in fp16 (|q - z| <= 255 <
// 2^11), and the fp16 product rounds the exact s (q - z) once.
template <int FMT>
__device__ __forceinline__ uint4 uniform_pair8(const uint32_t* w, int s0, int h,
                                               const __half2 (&zb)[2][2], __half2 scale) {
  uint32_t o[4];
#pragma unroll
  for (int ss = 0; ss < 2; ++ss)
#pragma unroll
    for (int dkp = 0; dkp < 2; ++dkp) {
      const int s = s0 + ss, r = h + 2 * dkp;
      const uint32_t f = code_fields<FMT>(w, s, r) | (magic_half(field_shift<FMT>(s, r)) * 0x10001u);
      const __half2 d = __hsub2(u32_as_h2(f), zb[s & 1][h]);
      o[2 * ss + dkp] = h2_as_u32(__hmul2(d, scale));
    }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// LUT4: the eight weights fp16(fp32(lut[q]) * absmax) of steps s0, s0 + 1 for row half h,
// with the product rounded to fp32 first.  Byte r of word s holds the two codes of
// fragment register r (low nibble = the smaller k); `a` is the absmax of the row half's
// 64-element block.
__device__ __forceinline__ uint4 lut_pair8(const uint32_t* w, int s0, int h, const float* lut_s,
                                           float a) {
  uint32_t o[4];
#pragma unroll
  for (int ss = 0; ss < 2; ++ss)
#pragma unroll
    for (int dkp = 0; dkp < 2; ++dkp) {
      const int s = s0 + ss, r = h + 2 * dkp;
      const uint32_t byte = (w[s] >> (8 * r)) & 0xFFu;
      const float lo = __fmul_rn(lut_s[byte & 0xFu], a);
      const float hi = __fmul_rn(lut_s[byte >> 4], a);
      o[2 * ss + dkp] = h2_as_u32(__floats2half2_rn(lo, hi));
    }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace qdq
