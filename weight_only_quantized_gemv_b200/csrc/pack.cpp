// Host-side packer: canonical code / parameter / Tile-COO layouts -> kernel layout.
// Plain C++ on host memory, no CUDA calls.  The layout itself is described in layout.h.
#include <stdint.h>
#include <string.h>

#include <vector>

#include "layout.h"
#include "qlinear.h"

using namespace qlayout;

namespace {

bool fmt_ok(int fmt) {
  return fmt == kW2 || fmt == kW3 || fmt == kW4 || fmt == kW8 || fmt == kLUT4;
}

bool shape_ok(int N, int K) {
  return N >= kTileN && K >= kGroup && N % kTileN == 0 && K % kGroup == 0;
}

// Code of weight (k, n) in the canonical layout.
inline uint32_t canonical_code(int fmt, const void* canon, int N, int k, int n) {
  if (fmt == kLUT4) {
    const uint8_t* b = static_cast<const uint8_t*>(canon);
    const uint8_t v = b[(size_t)(k >> 1) * N + n];
    return (k & 1) ? (v >> 4) : (v & 0xF);
  }
  // each column's words are one little-endian bit stream: code k in bits [b k, b k + b)
  const int bits = fmt;
  const uint32_t* w = static_cast<const uint32_t*>(canon);
  const long long o = (long long)bits * k;
  const long long j = o >> 5;
  const int sh = (int)(o & 31);
  uint64_t v = w[(size_t)j * N + n];
  if (sh + bits > 32) v |= (uint64_t)w[(size_t)(j + 1) * N + n] << 32;
  return (uint32_t)(v >> sh) & ((1u << bits) - 1);
}

}  // namespace

extern "C" size_t qlinear_packed_bytes(int fmt, int N, int K) {
  if (!fmt_ok(fmt) || !shape_ok(N, K)) return 0;
  return (size_t)N * K * code_bits(fmt) / 8;
}

extern "C" size_t qlinear_params_bytes(int fmt, int N, int K) {
  if (!fmt_ok(fmt) || !shape_ok(N, K)) return 0;
  if (fmt == kLUT4) return (size_t)(K / kLutBlock) * N * sizeof(float);
  return (size_t)(K / kGroup) * N * sizeof(uint16_t);
}

extern "C" ql_status qlinear_pack(int fmt, const void* canonical, void* packed, int N, int K) {
  if (!fmt_ok(fmt)) return QL_ERR_UNSUPPORTED;
  if (!canonical || !packed) return QL_ERR_NULL;
  if (!shape_ok(N, K)) return QL_ERR_SHAPE;
  const int G = K / kGroup;
  const int ntiles = N / kTileN;
  const int nblocks = (ntiles + kBlockTiles - 1) / kBlockTiles;
  const int WL = words_per_lane(fmt);
  uint32_t* out = static_cast<uint32_t*>(packed);
#pragma omp parallel for schedule(dynamic, 1)
  for (int b = 0; b < nblocks; ++b) {
    const int tb = tiles_in_block(b, ntiles);
    for (int g = 0; g < G; ++g) {
      for (int jj = 0; jj < tb; ++jj) {
        uint32_t* chunk = out + chunk_index(b, g, jj, G, ntiles) * 32 * WL;
        const int n_base = (b * kBlockTiles + jj) * kTileN;
        for (int lane = 0; lane < 32; ++lane) {
          const int gi = lane >> 2, t = lane & 3;
          uint32_t words[16] = {0};
          for (int s = 0; s < 8; ++s)
            for (int dk = 0; dk < 4; ++dk)
              for (int r8 = 0; r8 <= 8; r8 += 8) {
                const int k = g * kGroup + k_in_group(s, t, dk);
                const int n = n_base + gi + r8;
                int wi, bit;
                const uint32_t q = canonical_code(fmt, canonical, N, k, n);
                if (fmt == kW3) {  // low two bits as a W2 code, high bit in its own plane
                  code_position(kW2, s, dk, r8, &wi, &bit);
                  words[wi] |= (q & 3u) << bit;
                  code_position_w3_high(s, dk, r8, &wi, &bit);
                  words[wi] |= (q >> 2) << bit;
                } else {
                  code_position(fmt, s, dk, r8, &wi, &bit);
                  words[wi] |= q << bit;
                }
              }
          for (int w = 0; w < WL; ++w) chunk[word_index_fmt(fmt, w, lane)] = words[w];
        }
      }
    }
  }
  return QL_OK;
}

extern "C" ql_status qlinear_pack_params(int fmt, const void* canonical, void* packed, int N, int K) {
  if (!fmt_ok(fmt)) return QL_ERR_UNSUPPORTED;
  if (!canonical || !packed) return QL_ERR_NULL;
  if (!shape_ok(N, K)) return QL_ERR_SHAPE;
  const int G = K / kGroup;
  const int ntiles = N / kTileN;
  const int nblocks = (ntiles + kBlockTiles - 1) / kBlockTiles;
  for (int b = 0; b < nblocks; ++b) {
    const int tb = tiles_in_block(b, ntiles);
    for (int g = 0; g < G; ++g)
      for (int jj = 0; jj < tb; ++jj) {
        const long long c = chunk_index(b, g, jj, G, ntiles);
        const int n_base = (b * kBlockTiles + jj) * kTileN;
        for (int gi = 0; gi < 8; ++gi)
          for (int h = 0; h < 2; ++h) {
            const int n = n_base + gi + 8 * h;
            if (fmt == kLUT4) {
              const float* a = static_cast<const float*>(canonical);
              float* o = static_cast<float*>(packed);
              for (int blk = 0; blk < 2; ++blk)
                o[c * 32 + gi * 4 + blk * 2 + h] = a[(size_t)(2 * g + blk) * N + n];
            } else {
              const uint16_t* a = static_cast<const uint16_t*>(canonical);
              uint16_t* o = static_cast<uint16_t*>(packed);
              o[c * 16 + gi * 2 + h] = a[(size_t)g * N + n];
            }
          }
      }
  }
  return QL_OK;
}

// Codebook indices (canonical uint8 [K / 4][N]: the code of the 4-vector k = 4j .. 4j + 3 of
// column n) into the tensor-core GEMV layout: chunks (block, group, tile) in the order of the
// uniform formats, 512 bytes each, lane l's 16 bytes at 16 l; byte 2 s + r8 holds the code of
// row 16 tile + gi + 8 r8 for step s, whose k are 128 g + k_in_group(s, t, 0 .. 3) (one whole
// vector, since k_in_group(s, t, 0) is a multiple of 4).
extern "C" ql_status qlinear_pack_codebook_tc(const uint8_t* codes, uint8_t* packed, int N, int K) {
  if (!codes || !packed) return QL_ERR_NULL;
  if (!shape_ok(N, K)) return QL_ERR_SHAPE;
  const int G = K / kGroup;
  const int ntiles = N / kTileN;
  const int nblocks = (ntiles + kBlockTiles - 1) / kBlockTiles;
#pragma omp parallel for schedule(dynamic, 1)
  for (int b = 0; b < nblocks; ++b) {
    const int tb = tiles_in_block(b, ntiles);
    for (int g = 0; g < G; ++g)
      for (int jj = 0; jj < tb; ++jj) {
        uint8_t* chunk = packed + chunk_index(b, g, jj, G, ntiles) * 512;
        const int n_base = (b * kBlockTiles + jj) * kTileN;
        for (int lane = 0; lane < 32; ++lane) {
          const int gi = lane >> 2, t = lane & 3;
          for (int s = 0; s < 8; ++s)
            for (int r8 = 0; r8 < 2; ++r8) {
              const int j = (g * kGroup + k_in_group(s, t, 0)) / 4;
              chunk[lane * 16 + 2 * s + r8] = codes[(size_t)j * N + n_base + gi + 8 * r8];
            }
        }
      }
  }
  return QL_OK;
}

// Reorder Tile-COO tiles from the canonical K-major tile order (t = kt * NB + nt) to
// the order the fused kernel walks them (t' = nt * (K / 128) + kt), so the outliers
// of one run of work units are contiguous.  Entries keep their in-tile order.
extern "C" ql_status qlinear_pack_tilecoo(const uint32_t* offsets, const uint8_t* rc,
                                          const uint16_t* vals, int N, int K,
                                          uint32_t* offsets_out, uint8_t* rc_out,
                                          uint16_t* vals_out) {
  if (!offsets || !rc || !vals || !offsets_out || !rc_out || !vals_out) return QL_ERR_NULL;
  if (N <= 0 || K <= 0 || N % 128 || K % 128) return QL_ERR_SHAPE;
  const int NB = N / 128, KT = K / 128;
  const long long T = (long long)NB * KT;
  if (offsets[0] != 0) return QL_ERR_SHAPE;
  for (long long t = 0; t < T; ++t)
    if (offsets[t + 1] < offsets[t]) return QL_ERR_SHAPE;
  uint32_t pos = 0;
  offsets_out[0] = 0;
  for (int nt = 0; nt < NB; ++nt)
    for (int kt = 0; kt < KT; ++kt) {
      const long long t = (long long)kt * NB + nt;
      const uint32_t b = offsets[t], e = offsets[t + 1];
      const uint32_t n = e - b;
      memcpy(rc_out + 2 * (size_t)pos, rc + 2 * (size_t)b, 2 * (size_t)n);
      memcpy(vals_out + pos, vals + b, sizeof(uint16_t) * n);
      pos += n;
      offsets_out[(long long)nt * KT + kt + 1] = pos;
    }
  return QL_OK;
}

// Sub-groups per 128-k unit for a group size: 4 (g = 32), 2 (64), 1 (128, or per-channel
// g = K, whose one parameter per column is repeated in every 128-k unit); 0 if unsupported.
static int subgroups(int group, int K) {
  if (group == 32) return 4;
  if (group == 64) return 2;
  if (group == kGroup || group == K) return 1;
  return 0;
}

extern "C" size_t qlinear_params_bytes_grouped(int fmt, int group, int N, int K) {
  if (fmt != kW2 && fmt != kW3 && fmt != kW4 && fmt != kW8) return 0;
  if (!shape_ok(N, K) || !subgroups(group, K)) return 0;
  if (fmt == kW3 && subgroups(group, K) != 1) return 0;  // W3: group 128 or per-channel
  return (size_t)(K / kGroup) * subgroups(group, K) * N * sizeof(uint16_t);
}

extern "C" ql_status qlinear_pack_params_grouped(int fmt, int group, const void* canonical,
                                                 void* packed, int N, int K) {
  if (fmt != kW2 && fmt != kW3 && fmt != kW4 && fmt != kW8) return QL_ERR_UNSUPPORTED;
  if (!canonical || !packed) return QL_ERR_NULL;
  const int NS = subgroups(group, K);
  if (!shape_ok(N, K) || !NS || (fmt == kW3 && NS != 1)) return QL_ERR_SHAPE;
  const bool per_channel = group == K && group != kGroup;
  const int G = K / kGroup;
  const int ntiles = N / kTileN;
  const int nblocks = (ntiles + kBlockTiles - 1) / kBlockTiles;
  const uint16_t* a = static_cast<const uint16_t*>(canonical);
  uint16_t* o = static_cast<uint16_t*>(packed);
  for (int b = 0; b < nblocks; ++b) {
    const int tb = tiles_in_block(b, ntiles);
    for (int g = 0; g < G; ++g)
      for (int jj = 0; jj < tb; ++jj) {
        const long long c = chunk_index(b, g, jj, G, ntiles);
        const int n_base = (b * kBlockTiles + jj) * kTileN;
        for (int ss = 0; ss < NS; ++ss)
          for (int gi = 0; gi < 8; ++gi)
            for (int h = 0; h < 2; ++h) {
              const int n = n_base + gi + 8 * h;
              const int src_group = per_channel ? 0 : g * NS + ss;
              o[(c * NS + ss) * 16 + gi * 2 + h] = a[(size_t)src_group * N + n];
            }
      }
  }
  return QL_OK;
}
