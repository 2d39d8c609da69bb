// Kernel-side data layout shared by the host packer and the device kernels.
//
// Work grid.  The output columns are cut into 16-column tiles (the row dimension
// of one m16n8k16 tensor-core fragment) and the tiles into 128-column blocks of
// up to 8 tiles; K is cut into 128-element groups (the quantization group).  A
// (block, group) pair is one work unit: 128 x 128 weights, which is also one
// Tile-COO outlier tile.  A "chunk" is one (tile, group): 16 x 128 weights, read
// by one warp as one coalesced load per lane.
//
// Chunk order in memory: block-major, then group, then tile inside the block,
//   chunk(b, g, jj) = b * G * 8 + g * TB(b) + jj,   TB(b) = tiles in block b,
// so the units of one block sit back to back and a CTA that walks a run of
// units reads one contiguous byte range.  Only the last block may hold fewer
// than 8 tiles.
//
// Inside a chunk the words of each lane are stored as 16-byte quads: word w of lane
// l sits at 32-bit index ((w / 4) * 32 + l) * 4 + w % 4, so that one 128-bit access
// of a whole warp covers 512 contiguous bytes (coalesced in global memory,
// conflict-free in shared memory).
//
// Every lane (gi = lane / 4, t = lane % 4) owns the A fragment of
// tensor-core step s (s = 0..7, 16 K each): rows gi and gi + 8 of the tile and
// the K slots {2t, 2t+1, 2t+8, 2t+9}.  The packer maps those slots to the four
// consecutive k = 128 g + 32 (s / 2) + 8 t + 4 (s % 2) + dk, dk = 0..3, so that
// the matching x fragment of a lane is one 16-byte load of x[m][k .. k + 7]
// covering two steps.  Slot 2t <-> dk 0, 2t+1 <-> dk 1, 2t+8 <-> dk 2,
// 2t+9 <-> dk 3.
//
// Bit position of the code of (step s, dk, row half r8 in {0, 8}) in the lane's
// words (fields chosen so that AND masks yield fp16 pairs with the code in the
// low mantissa bits, i.e. the exact subnormal code * 2^-24 * 2^shift):
//   W4  : word s,            bit 16 (dk & 1) + 8 (dk >> 1) + 4 (r8 / 8)
//   W2  : word s / 2,        bit 16 (dk & 1) + 8 (dk >> 1) + 2 (r8 / 8) + 4 (s & 1)
//   W8  : word 2 s + r8 / 8, bit 16 (dk & 1) + 8 (dk >> 1)
//   LUT4: word s,            bit 16 (dk >> 1) + 8 (r8 / 8) + 4 (dk & 1)
//         (each byte holds the two codes of one fragment register)
//   W3  : two bit planes, q = q2 + 4 q1.  The low two bits q2 sit exactly where W2 puts a
//         2-bit code (words 0..3, the quad of the lane); the high bit q1 sits in word
//         4 + s / 4, bit 16 (dk & 1) + 4 (s % 4) + r8 / 8 + 2 (dk >> 1), so that shifting
//         the word right by 4 (s % 4) + r (r = the fragment register) and masking bits
//         0 and 16 yields register r of step s.  Words 4 and 5 of a lane are not in the
//         quad layout: they follow the 512 bytes of quads, 8 bytes per lane (a 768-byte
//         chunk).
//
// Parameters follow the chunk order: per chunk, for gi = 0..7 the pair of
// columns (gi, gi + 8):
//   scales / zeros (fp16): [chunk][gi][r8 / 8]                 16 per chunk
//   LUT4 absmax (fp32)   : [chunk][gi][64-block 0..1][r8 / 8]  32 per chunk
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define QL_HD __host__ __device__ __forceinline__
#else
#define QL_HD inline
#endif

namespace qlayout {

// kCB: a codebook of 256 fp16 4-vectors with 8-bit codes (m1v4g128) in the tensor-core GEMV
// layout: per chunk lane, the code of each (step, row half) in one byte (2 s + r8)
enum { kW2 = 2, kW3 = 3, kW4 = 4, kW8 = 8, kLUT4 = 16, kCB = 32 };

constexpr int kGroup = 128;      // quantization group along K (uniform formats)
constexpr int kLutBlock = 64;    // absmax block along K (LUT4)
constexpr int kTileN = 16;       // columns per tile
constexpr int kBlockTiles = 8;   // tiles per block (128 columns)

// 32-bit words of codes per lane per chunk.
QL_HD int words_per_lane(int fmt) {
  return (fmt == kW2 || fmt == kCB) ? 4 : fmt == kW3 ? 6 : fmt == kW8 ? 16 : 8;
}
QL_HD int chunk_bytes(int fmt) { return 128 * words_per_lane(fmt); }
QL_HD int code_bits(int fmt) { return fmt == kLUT4 ? 4 : fmt; }

// 32-bit index, inside its chunk, of word w of lane l
QL_HD int word_index(int w, int lane) { return ((w >> 2) * 32 + lane) * 4 + (w & 3); }

// ... for a format: W3's high-bit words 4 and 5 follow the quads, two per lane
QL_HD int word_index_fmt(int fmt, int w, int lane) {
  return (fmt == kW3 && w >= 4) ? 128 + 2 * lane + (w - 4) : word_index(w, lane);
}

QL_HD int tiles_in_block(int b, int ntiles) {
  int r = ntiles - kBlockTiles * b;
  return r < kBlockTiles ? r : kBlockTiles;
}

QL_HD long long chunk_index(int b, int g, int jj, int G, int ntiles) {
  return (long long)b * G * kBlockTiles + (long long)g * tiles_in_block(b, ntiles) + jj;
}

// k offset inside the group of (step s, lane t, dk)
QL_HD int k_in_group(int s, int t, int dk) { return 32 * (s >> 1) + 8 * t + 4 * (s & 1) + dk; }

// (word index, bit position) of the code of (step s, dk, r8) for a lane.
QL_HD void code_position(int fmt, int s, int dk, int r8, int* word, int* bit) {
  const int hi = r8 >> 3;
  switch (fmt) {
    case kW4:
      *word = s;
      *bit = 16 * (dk & 1) + 8 * (dk >> 1) + 4 * hi;
      break;
    case kW2:
      *word = s >> 1;
      *bit = 16 * (dk & 1) + 8 * (dk >> 1) + 2 * hi + 4 * (s & 1);
      break;
    case kW8:
      *word = 2 * s + hi;
      *bit = 16 * (dk & 1) + 8 * (dk >> 1);
      break;
    default:  // LUT4
      *word = s;
      *bit = 16 * (dk >> 1) + 8 * hi + 4 * (dk & 1);
      break;
  }
}

// W3: (word, bit) of the high bit q1 of (step s, dk, r8); q2 takes code_position(kW2, ...)
QL_HD void code_position_w3_high(int s, int dk, int r8, int* word, int* bit) {
  *word = 4 + (s >> 2);
  *bit = 16 * (dk & 1) + 4 * (s & 3) + (r8 >> 3) + 2 * (dk >> 1);
}

}  // namespace qlayout
