/*
 * qlinear.h -- C ABI of the weight-only-quantized linear layer for NVIDIA B200 (sm_100a).
 *
 *   y[M, N] = x[M, K] . dequant(Wq)[K, N],   M = 1..16 activation rows (LLM decoding)
 *
 * Also: a prefill path for any M (stand-alone dequantization to fp16 + one dense GEMM), a
 * measured policy map with a dispatcher for any M, and a codebook GEMV with a Psumbook
 * (sections further down).
 *
 * Formats
 *   W2 / W3 / W4 / W8 : group-wise asymmetric uniform codes, one fp16 scale s and one
 *                  fp16 zero z (an integer) per 128-element group along K per
 *                  column; w = s * (q - z).  Sources: QFactory (ATC'25) page,
 *                  "问题与动机" and observation 1 (fine-grained asymmetric group-wise
 *                  quantization, group size 128, W8/W4/W2).
 *   LUT4         : 4-bit indices into a 16-entry fp16 table with an fp32 absmax per
 *                  64-element block along K per column; w = lut[q] * absmax.
 *                  Source: "Fast NF4 Dequantization Kernels for Large Language Model
 *                  Inference" page, abstract and method section (NF4 lookup table).
 *   W4 + outliers: W4 dense part plus fp16 outliers in Tile-COO (128 x 128 K x N
 *                  tiles, uint32 per-tile offsets, uint8 in-tile (row, col) pairs);
 *                  y = x . dequant(W_dense) + x . W_outlier.  Source: FlashQuant page,
 *                  English abstract (fused dense GEMM + sparse outlier path, sparse-
 *                  dense tiling, Tile-COO encoding).
 *
 * Every GEMV uses the deferred-dequantization identity of the QFactory page
 * (observation 2, J-matrix expansion, Table 2) in its weight-only form:
 *   y[m, n] = sum_g s[g, n] * ( sum_{k in g} q[k, n] x[m, k] - z[g, n] * sum_{k in g} x[m, k] ).
 *
 * Conventions (all entry points)
 *   - fp16 arguments are IEEE binary16 bit patterns (uint16_t); fp32 are IEEE binary32.
 *   - "device" pointers point to memory of the current CUDA device, owned by the caller;
 *     the library never allocates, frees or synchronizes.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream); device work is enqueued
 *     asynchronously on it and the call returns without waiting.
 *   - The return value is a ql_status.  Argument errors are detected on the host before
 *     anything is enqueued; QL_ERR_CUDA reports a launch failure (cudaGetLastError).
 *   - Shapes: K % 128 == 0, N % 16 == 0, 1 <= M <= 16; the outlier variant also needs
 *     N % 128 == 0.  All 2-bit shapes with K % 128 == 0 are accepted.
 *   - Group sizes (W2 / W4 / W8 entries, `group` argument): 128; 64 and 32 (finer groups,
 *     parameters packed by qlinear_pack_params_grouped; QFactory page, "问题与动机" and
 *     Differentiated Qtile Scheduling: fine-grained groups, their parameters reused from
 *     registers); K (per-channel: one scale and zero per column, repeated per 128-k unit by
 *     qlinear_pack_params_grouped, then read like group 128).  LUT4 (block 64), the outlier
 *     variant and qlinear_w4a16_noalloc take their fixed block / group only.
 *   - Calls are thread-safe; two calls that share one workspace must not overlap in time
 *     (issue them on one stream).
 *
 * Canonical (packer input) layouts, host memory:
 *   uniform codes : uint32[K * bits / 32][N]; each column's words form one little-endian bit
 *                   stream along K (word j = stream bits 32 j .. 32 j + 31) and the code of
 *                   weight (k, n) is stream bits [bits*k, bits*k + bits).  For 2, 4, 8 bits:
 *                   word (j, n) bits [bits*i, bits*i + bits) hold weight (P*j + i, n),
 *                   P = 32 / bits; 3-bit codes (W3) straddle words, 32 codes per 3 words
 *   scales, zeros : fp16 [K / 128][N]
 *   LUT4 codes    : uint8 [K / 2][N]; low nibble = even k, high nibble = odd k
 *   LUT4 absmax   : fp32 [K / 64][N];  lut: fp16 [16]
 *   Tile-COO      : tiles t = kt * (N / 128) + nt; offsets uint32[T + 1] (offsets[0] = 0,
 *                   offsets[T] = nnz); rc uint8[nnz][2] = (k - 128 kt, n - 128 nt);
 *                   vals fp16[nnz].  The kernels read this layout directly.
 */
#ifndef QLINEAR_H_
#define QLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QL_OK = 0,
  QL_ERR_NULL = 1,        /* a required pointer is NULL */
  QL_ERR_SHAPE = 2,       /* M, N, K, group or block outside the supported set */
  QL_ERR_ALIGN = 3,       /* a pointer is not aligned as documented */
  QL_ERR_UNSUPPORTED = 4, /* unknown format */
  QL_ERR_WORKSPACE = 5,   /* workspace missing or smaller than qlinear_workspace_bytes() */
  QL_ERR_CUDA = 6,        /* a CUDA runtime call or kernel launch failed */
  QL_ERR_LIBRARY = 7      /* reserved (no library is opened at run time) */
} ql_status;

typedef enum {
  QL_FMT_W2 = 2,
  QL_FMT_W3 = 3,
  QL_FMT_W4 = 4,
  QL_FMT_W8 = 8,
  QL_FMT_LUT4 = 16,
  QL_FMT_CB = 32 /* m1v4g128 codebook, tensor-core layout (qlinear_codebook_tc): for
                    qlinear_workspace_bytes and qlinear_plan only */
} ql_format;

/* Opaque stream handle, ABI-compatible with cudaStream_t. */
typedef struct CUstream_st* ql_stream_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* ql_status_str(int status);

/* ---------------------------------------------------------------------------
 * Host-side packer.  Host pointers, caller-allocated outputs, no device work.
 * The packed codes have exactly the byte count of the canonical codes; the packed
 * quantization parameters have exactly the byte count of the canonical ones.
 * ------------------------------------------------------------------------- */

/* Bytes of packed codes (= canonical code bytes, K * N * bits / 8); 0 on a bad shape. */
size_t qlinear_packed_bytes(int fmt, int N, int K);

/* Bytes of packed parameters: scales or zeros (fp16, K/128 * N each) for W2/W4/W8,
 * absmax (fp32, K/64 * N) for LUT4; 0 on a bad shape. */
size_t qlinear_params_bytes(int fmt, int N, int K);

/* Reorder canonical codes into the kernel layout (a bijection on code fields):
 * each warp of the GEMV then issues one 128/256-bit coalesced load per 16-column
 * tile and 128-element group, and each code lands where the tensor-core fragment
 * wants it.  `canonical` and `packed` are host buffers of qlinear_packed_bytes(). */
ql_status qlinear_pack(int fmt, const void* canonical, void* packed, int N, int K);

/* Reorder one canonical parameter array into the kernel layout: call it for the
 * scales and again for the zeros of W2/W4/W8 (fp16 [K/128][N]), or for the absmax of
 * LUT4 (fp32 [K/64][N]).  Host buffers of qlinear_params_bytes(). */
ql_status qlinear_pack_params(int fmt, const void* canonical, void* packed, int N, int K);

/* Bytes of packed scales (or zeros) for group size `group` of W2 / W4 / W8: K / 128 * NS * N
 * fp16, NS = 128 / group for groups 32 and 64, 1 for 128 and for per-channel (group = K);
 * 0 for other formats, groups or shapes. */
size_t qlinear_params_bytes_grouped(int fmt, int group, int N, int K);

/* Reorder one canonical parameter array (fp16 [K / group][N]; [1][N] for group = K) into
 * the kernel layout for that group size: per chunk, per sub-group, for gi = 0..7 the pair
 * of columns (gi, gi + 8).  Per-channel parameters are repeated in every 128-k unit.  Host
 * buffers; the output holds qlinear_params_bytes_grouped() bytes. */
ql_status qlinear_pack_params_grouped(int fmt, int group, const void* canonical, void* packed,
                                      int N, int K);

/* Reorder canonical Tile-COO (tiles numbered t = kt * (N/128) + nt) into the order the
 * fused outlier kernel walks them, t' = nt * (K/128) + kt, so that the outliers of one run
 * of (block, group) work units are contiguous.  Entries keep their in-tile order.  Host
 * buffers: offsets uint32[T+1] in and out, rc uint8[nnz][2], vals fp16[nnz].
 * Returns QL_ERR_SHAPE for N or K not multiples of 128 or non-monotone offsets. */
ql_status qlinear_pack_tilecoo(const uint32_t* offsets, const uint8_t* rc, const uint16_t* vals,
                               int N, int K, uint32_t* offsets_out, uint8_t* rc_out,
                               uint16_t* vals_out);

/* ---------------------------------------------------------------------------
 * Workspace.  The split-K fix-up needs fp32 partial sums and per-tile arrival
 * counters.  The caller allocates qlinear_workspace_bytes() on the device (256-byte
 * aligned) and zero-fills it ONCE before its first use; every completed call leaves
 * the counters at zero again, so no per-call clearing is needed.
 * ------------------------------------------------------------------------- */

/* Workspace bytes for a call with these arguments on the current device; 0 for invalid
 * arguments or when no CUDA device is available. */
size_t qlinear_workspace_bytes(int fmt, int M, int N, int K);

/* The first 32-bit word of a workspace collects sticky error flags of the calls that used
 * it: bit 0 = a consumer gave up waiting for a shared-memory stage, bit 1 = the producer
 * gave up waiting for a stage to be released (each wait is bounded so that a lost copy
 * cannot hang the GPU; results of such a call are undefined).  This call waits for
 * `stream`, copies the word to *flags and clears it.  Synchronous. */
ql_status qlinear_read_error(void* workspace, uint32_t* flags, ql_stream_t stream);

/* Failure-detection tests of the GEMV entries' bounded waits (the QFactory page's critical
 * analysis notes that the method leaves failure handling open; this is the library's own).
 * Process-wide settings read by every later GEMV call:
 *   wait_limit        : try_wait rounds after which a stage wait sets its flag
 *                       (1 = copy landed late, 2 = stage released late) and then waits at
 *                       most 2^22 more rounds; 0 restores the default 2^22
 *   producer_delay_us : CTA 0's producer waits this long before its first copy
 *   consumer_hold_us  : CTA 0's first consumer warp holds its first stage this long
 *                       before releasing it
 * Delays are at most 65535 us (QL_ERR_SHAPE otherwise); (0, 0, 0) restores normal
 * operation.  A delay shorter than the second wait gives flagged calls with correct
 * results.  While a setting is active, the W4 kernels for M = 1 and M = 9..16 run as
 * instances compiled with these hooks (the other kernels keep their fixed 2^22-round limit
 * and no hooks).  Not thread-safe with respect to concurrent GEMV calls' settings. */
ql_status qlinear_debug_wait_test(uint32_t wait_limit, uint32_t producer_delay_us,
                                  uint32_t consumer_hold_us);

/* ---------------------------------------------------------------------------
 * Hot path (device pointers, asynchronous on `stream`).
 *   x       : fp16 [M][K] row-major, 16-byte aligned
 *   qweight : packed codes from qlinear_pack, 32-byte aligned
 *   scales, zeros : packed fp16 parameters from qlinear_pack_params (group 128) or
 *             qlinear_pack_params_grouped (group 64, 32 or K), 16-byte aligned
 *   y       : fp16 [M][N] row-major output (round-to-nearest-even of an fp32 sum)
 *   group   : W2 / W4 / W8: 128, 64, 32 or K (per-channel); W3: 128 or K; the outlier
 *             variant and qlinear_w4a16_noalloc: 128 (QL_ERR_SHAPE otherwise)
 * ------------------------------------------------------------------------- */

ql_status qlinear_w4a16(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                        const uint16_t* zeros, uint16_t* y, int M, int N, int K, int group,
                        void* workspace, size_t workspace_bytes, ql_stream_t stream);

ql_status qlinear_w2a16(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                        const uint16_t* zeros, uint16_t* y, int M, int N, int K, int group,
                        void* workspace, size_t workspace_bytes, ql_stream_t stream);

ql_status qlinear_w8a16(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                        const uint16_t* zeros, uint16_t* y, int M, int N, int K, int group,
                        void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* 3-bit codes (QFactory page, observation 1: bit widths below 4 raise the parameter share).
 * Packed by qlinear_pack(QL_FMT_W3, ...) into two planes: the low two bits of each code
 * where W2 puts its codes, the high bit in a separate plane (768 bytes per 16 x 128 chunk),
 * and evaluated as sum q x = sum q2 x + 4 sum q1 x (two tensor-core steps per k-step).
 * Arguments as qlinear_w4a16; group 128 or per-channel (group = K) only.  W3 has no prefill,
 * policy-map or no-alloc entry. */
ql_status qlinear_w3a16(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                        const uint16_t* zeros, uint16_t* y, int M, int N, int K, int group,
                        void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* LUT4: codes packed by qlinear_pack(QL_FMT_LUT4), 32-byte aligned; lut16: fp16[16]
 * (device); absmax packed by qlinear_pack_params(QL_FMT_LUT4), 16-byte aligned;
 * block must be 64. */
ql_status qlinear_lut4(const uint16_t* x, const uint8_t* codes, const uint16_t* lut16,
                       const float* absmax, uint16_t* y, int M, int N, int K, int block,
                       void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* W4 dense part (as qlinear_w4a16) plus the Tile-COO outliers, processed in the same
 * kernel.  The Tile-COO arrays are those written by qlinear_pack_tilecoo (tiles in
 * block-major order): tile_offsets uint32[T+1] (4-byte aligned), tile_rc uint8[nnz][2]
 * (2-byte aligned), tile_vals fp16[nnz] (2-byte aligned), T = (K/128) * (N/128).
 * Needs N % 128 == 0.  The dense code of every outlier position should
 * hold its group's zero code (then the dense part contributes nothing there).
 * The offsets must be non-decreasing with tile_offsets[T] = nnz (qlinear_pack_tilecoo
 * checks this; the hot path reads them as given).  In-tile rows and columns are taken
 * modulo 128, so a malformed pair gives a wrong sum, never an access outside the tile. */
ql_status qlinear_w4a16_outlier(const uint16_t* x, const uint32_t* qweight,
                                const uint16_t* scales, const uint16_t* zeros,
                                const uint32_t* tile_offsets, const uint8_t* tile_rc,
                                const uint16_t* tile_vals, uint16_t* y, int M, int N, int K,
                                int group, void* workspace, size_t workspace_bytes,
                                ql_stream_t stream);

/* The W4A16 GEMV of qlinear_w4a16 for callers that cannot allocate device memory (e.g. a
 * plug-in whose device memory belongs to a host application or a fixed pool, or code that
 * must not call cudaMalloc/cudaFree because they synchronize or are not allowed where it
 * runs).  No page describes this entry; it has no counterpart in the method.
 * Same arguments as qlinear_w4a16 without the workspace: the split-K scratch is a fixed
 * 8 MiB array inside the library (on every device, from library load to process exit).
 * It allocates nothing and frees nothing.  Returns QL_ERR_WORKSPACE if a call would need
 * more than that scratch.  The first call on a device looks up the scratch's device
 * address (make it before any stream capture); it is looked up again when the device's
 * context changes (a device reset may move the array).  Every call on a device shares
 * the scratch: calls whose device work overlaps in time race and must not be issued.
 * Each call clears its arrival counters on `stream` before its launch, after every
 * argument check (a rejected call enqueues nothing).  A device wait that gives up sets
 * a flag in the scratch's error word, which stays set until
 * qlinear_w4a16_noalloc_read_error reads it. */
ql_status qlinear_w4a16_noalloc(const uint16_t* x, const uint32_t* qweight,
                                const uint16_t* scales, const uint16_t* zeros, uint16_t* y,
                                int M, int N, int K, int group, ql_stream_t stream);

/* The error word of qlinear_w4a16_noalloc's scratch on the current device (the flags of
 * qlinear_read_error), then cleared.  Waits for `stream`; synchronous.  Allocates
 * nothing.  No page describes this entry; it has no counterpart in the method. */
ql_status qlinear_w4a16_noalloc_read_error(uint32_t* flags, ql_stream_t stream);

/* ---------------------------------------------------------------------------
 * Prefill (M >> 16): stand-alone dequantization to fp16, then one dense GEMM.
 * Source: "Fast NF4 Dequantization Kernels for Large Language Model Inference" page,
 * method section (technical framework: load the codes, dequantize, write FP16 back to
 * global memory for the following matmul; the 16-entry table lives in 64 bytes of
 * shared memory); QFactory page, assumption stress test and limitation 1 (prefill and
 * large batches are compute-bound, where the fused GEMV stops paying).
 * ------------------------------------------------------------------------- */

/* Dequantize packed weights into a dense fp16 matrix w[N][K] (row n = output column n,
 * row stride K: the weight layout of a linear layer).  Device pointers, asynchronous on
 * `stream`.
 *   packed : packed codes (qlinear_pack), 16-byte aligned
 *   p0, p1 : W2/W4/W8: packed scales and zeros (fp16, 4-byte aligned; zeros are integers
 *            with |z| <= 1024);  LUT4: p0 = the fp16 lut[16] (2-byte aligned), p1 = the
 *            packed fp32 absmax (16-byte aligned)
 *   w      : fp16 [N][K], caller-allocated, 16-byte aligned, fully overwritten
 * Values: W2/W4/W8 give fp16(s * (q - z)), the exact product rounded once to nearest even
 * (overflow gives +-inf); LUT4 gives fp16(fp32(lut[q]) * absmax), the fp32 product rounded
 * to fp32 and then to fp16.  N % 16 == 0, K % 128 == 0, N, K > 0 (QL_ERR_SHAPE otherwise). */
ql_status qlinear_dequant_fp16(int fmt, const void* packed, const void* p0, const void* p1,
                               uint16_t* w, int N, int K, ql_stream_t stream);

/* y[M][N] = x[M][K] . w_fp16[N][K]^T for any M >= 1: qlinear_dequant_fp16 into the caller's
 * w_fp16 (N * K * 2 bytes, 16-byte aligned, overwritten), then this library's tensor-core
 * GEMM on `stream` (tcgen05.mma with fp16 operands staged by TMA, fp32 accumulation in
 * tensor memory, fp16 round-to-nearest-even output).  x is an fp16 row-major device array,
 * 16-byte aligned (QL_ERR_ALIGN otherwise); y fp16 row-major, 2-byte aligned.  N % 16 == 0,
 * K % 128 == 0.  Device waits that run out are reported by qlinear_prefill_read_error. */
ql_status qlinear_prefill(int fmt, const uint16_t* x, const void* packed, const void* p0,
                          const void* p1, uint16_t* w_fp16, uint16_t* y, int M, int N, int K,
                          ql_stream_t stream);

/* The same product without the fp16 weight matrix: y[M][N] = x[M][K] . W^T with W the fp16
 * weights qlinear_dequant_fp16 would write, dequantized inside the GEMM (the NF4 page's
 * codes -> FP16 -> matmul, with FP16 kept in shared memory as the tensor cores' operand
 * instead of written back).  fmt W2 / W4 / W8 (group 128) or LUT4; packed, p0, p1 as for
 * qlinear_dequant_fp16 but 16-byte aligned (except the LUT, 2-byte); x 16-byte aligned, y
 * 2-byte aligned; any M >= 1, N % 16 == 0, K % 128 == 0.  Asynchronous on `stream`;
 * allocates nothing.
 *   workspace : NULL, or device memory of qlinear_prefill_workspace_bytes(M, N, K) bytes,
 *               16-byte aligned and zero-filled before its first use (the kernel leaves it
 *               zero again).  With a workspace the k-blocks of all output tiles are shared
 *               out evenly over one CTA per SM (stream-K: tiles split between CTAs meet in
 *               the workspace, summed in a fixed order, so results are reproducible);
 *               without one each CTA takes whole 128 x 256 (M > 128) or 128 x 128 tiles.
 *               QL_ERR_WORKSPACE if it is too small.  Calls sharing a workspace must not
 *               overlap in time. */
ql_status qlinear_prefill_fused(int fmt, const uint16_t* x, const void* packed, const void* p0,
                                const void* p1, uint16_t* y, int M, int N, int K,
                                void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* Bytes of the qlinear_prefill_fused workspace on the current device (0 for an unsupported
 * shape). */
size_t qlinear_prefill_workspace_bytes(int M, int N, int K);

/* Sticky flags of the prefill GEMM kernels' bounded waits on the current device (1: a
 * pipeline stage's wait ran out, 2: an accumulator's wait ran out; results of such a call
 * are undefined), then cleared.  Waits for `stream`; synchronous. */
ql_status qlinear_prefill_read_error(uint32_t* flags, ql_stream_t stream);

/* ---------------------------------------------------------------------------
 * Codebook GEMV with a Psumbook.  Source: CodeGEMM page (NeurIPS 2025 notes), method:
 * overall framework (build the Psumbook, look codes up, accumulate), key design one
 * (precomputed centroid . input partial sums kept in shared memory instead of the
 * codebook), key design four (group normalization); configuration m1v4g128 (one codebook,
 * 4-weight vectors, 8-bit codes: 2 bits per weight plus one fp16 scale per 128).
 *
 *   w[k][n] = s[k / 128][n] * C[code[k / 4][n]][k % 4]
 *   y[m][n] = sum_g s[g][n] * sum_{j in g} P[m][j][code[j][n]],  P[m][j][i] = sum_t C[i][t] x[m][4j + t]
 *
 * Canonical layouts (host): codes uint8 [K / 4][N] (code of the 4-vector k = 4j .. 4j + 3
 * of column n); scales fp16 [K / 128][N]; codebook fp16 [256][4] (used as is by the GEMV).
 * Shapes: N % 32 == 0, K % 128 == 0, 1 <= M <= 4.  The Psumbook entries and every sum are
 * fp32; y is rounded once to fp16.
 * ------------------------------------------------------------------------- */

/* Reorder canonical codes into the kernel layout: 32-column tiles by 128-k groups, each
 * (tile, group) chunk 1024 bytes in which lane l's 32 codes form two 16-byte quads.  Host
 * buffers of K / 4 * N bytes. */
ql_status qlinear_pack_codebook(const uint8_t* codes, uint8_t* packed, int N, int K);

/* Reorder canonical scales into chunk order, fp16 [tile][group][lane].  Host buffers of
 * K / 128 * N fp16. */
ql_status qlinear_pack_codebook_scales(const uint16_t* scales, uint16_t* packed, int N, int K);

/* Workspace bytes for qlinear_codebook (per-tile arrival counters and fp32 partial sums of
 * the K ranges); 0 for invalid shapes or without a device.  Zero-fill it once before its
 * first use; every completed call leaves the counters at zero. */
size_t qlinear_codebook_workspace_bytes(int M, int N, int K);

/* y[M][N] = x[M][K] . W.  Device pointers: x fp16 (2-byte aligned), codes and scales as
 * packed above (16- and 2-byte aligned), codebook fp16 [256][4] (8-byte aligned), y fp16.
 * The workspace (16-byte aligned) is needed when the K range is split across CTAs (any
 * K > 256 at M = 1, K > 128 otherwise).  Asynchronous on `stream`; results are bit-for-bit
 * reproducible (partials are summed in a fixed order). */
ql_status qlinear_codebook(const uint16_t* x, const uint8_t* codes, const uint16_t* scales,
                           const uint16_t* codebook, uint16_t* y, int M, int N, int K,
                           void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* The same product on the tensor cores, through the GEMV kernel (qlinear_w2a16's pipeline,
 * stream-K grid and split-K fix-up): the codebook's 256 vectors are copied 16 times into
 * shared memory, and each tensor-core step takes, per lane, one 8-byte vector for each of
 * its two weight rows as the A fragment (the step's four k per lane are one vector).  The
 * Psumbook form (qlinear_codebook) follows the CodeGEMM page; this form reaches the same
 * sums with one lookup per 4 weights and row instead of one per 4 weights, row and token,
 * which on B200 is the faster use of shared memory (measured).
 *   codes    : packed by qlinear_pack_codebook_tc, 32-byte aligned;
 *   scales   : fp16 [K / 128][N] packed by qlinear_pack_params(QL_FMT_W4, ...), 16-byte
 *              aligned (the uniform formats' scale layout);
 *   codebook : fp16 [256][4], 8-byte aligned;
 *   x, y     : as qlinear_w4a16 (M <= 16, N % 16 == 0, K % 128 == 0);
 *   workspace: qlinear_workspace_bytes(QL_FMT_CB, M, N, K) bytes, as for qlinear_w4a16.
 * fp32 accumulation, y rounded once to fp16; reproducible. */
ql_status qlinear_codebook_tc(const uint16_t* x, const uint8_t* codes, const uint16_t* scales,
                              const uint16_t* codebook, uint16_t* y, int M, int N, int K,
                              void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* Canonical codes uint8 [K / 4][N] into the layout of qlinear_codebook_tc: the chunk order
 * of the uniform formats (16-column tiles by 128-k groups), 512 bytes per chunk, lane l's
 * 16 bytes at 16 l, byte 2 s + r of them the code of step s for row (tile column) l / 4 + 8 r.
 * Host buffers of K / 4 * N bytes. */
ql_status qlinear_pack_codebook_tc(const uint8_t* codes, uint8_t* packed, int N, int K);

/* ---------------------------------------------------------------------------
 * Measured policy map and dispatcher.
 * Source: ADAngel page (awesome-system-papers, OSDI'26), core method: an offline script
 * times every candidate kernel with CUDA events over the (M, N, K) and bit-width
 * combinations of a model and keeps the fastest in a table (the oracle policy map); at run
 * time the dispatcher looks the shape and bit width up and calls that kernel.  The offline
 * script here is the Python package's `tune` module; the table is host memory owned by the
 * library (a copy of what qlinear_policy_set receives).
 * ------------------------------------------------------------------------- */

typedef enum {
  QL_STRATEGY_GEMV = 0,    /* the fused GEMV (over 16-row slices of x when M > 16) */
  QL_STRATEGY_PREFILL = 1  /* the tensor-core prefill GEMM (qlinear_prefill / _fused) */
} ql_strategy;

typedef struct {
  int fmt;             /* ql_format */
  int N, K;            /* layer shape, matched exactly */
  int m_lo, m_hi;      /* rows of x covered, inclusive, 1 <= m_lo <= m_hi */
  int strategy;        /* ql_strategy */
  int warps_per_unit;  /* GEMV: 0 = the planner's rule, else 1, 2 or 4 (honoured by the W4
                          kernels at M <= 8; other kernels have one variant) */
  int ctas;            /* GEMV: 0 = the planner's rule, else the grid size (clamped to the
                          number of work units) */
} ql_policy_entry;

/* Install a policy table (copied; n = 0 clears it).  The first entry that covers a call
 * decides it.  Entries apply to the plain formats, not to qlinear_w4a16_outlier.  A table
 * changes grid sizes, so query qlinear_workspace_bytes after installing it.  Returns
 * QL_ERR_UNSUPPORTED for an unknown format or strategy, QL_ERR_SHAPE for an invalid shape,
 * M range, warps_per_unit or ctas (nothing is installed then). */
ql_status qlinear_policy_set(const ql_policy_entry* entries, int n);

/* Number of installed entries. */
int qlinear_policy_size(void);

/* The decision for (fmt, M, N, K): the covering table entry (*from_table = 1), else the
 * built-in rule (*from_table = 0): the GEMV for M <= 64 with the planner's rules, prefill
 * above; out->m_lo / m_hi give the rule's M range.  from_table may be NULL. */
ql_status qlinear_policy_lookup(int fmt, int M, int N, int K, ql_policy_entry* out,
                                int* from_table);

/* y[M][N] = x[M][K] . dequant(W) for any M >= 1, by the policy's decision:
 *   GEMV    : the format's GEMV entry (qlinear_w4a16 ...) on each 16-row slice of x / y in
 *             turn, all with `workspace` (at least qlinear_workspace_bytes(fmt, min(M, 16), N,
 *             K) bytes);
 *   PREFILL : qlinear_prefill into w_fp16 (N * K fp16) when w_fp16 is given, else
 *             qlinear_prefill_fused without a workspace (whole tiles per CTA).
 * Arguments as in those entries (p0 / p1: scales / zeros, or lut16 / absmax for LUT4; group
 * 128, LUT block 64).  Returns the first non-OK status of the calls it makes. */
ql_status qlinear_matmul(int fmt, const uint16_t* x, const void* packed, const void* p0,
                         const void* p1, uint16_t* y, int M, int N, int K, void* workspace,
                         size_t workspace_bytes, uint16_t* w_fp16, ql_stream_t stream);

/* ---------------------------------------------------------------------------
 * Debug entries (device pointers, asynchronous).  They decode the packed layout
 * with the same fragment-extraction code the GEMV kernels use.
 *   qlinear_debug_unpack : codes uint8 [K][N] (canonical order, one code per byte)
 *   qlinear_debug_dequant: w fp32 [K][N]; p0 = packed scales (fp16) or the device
 *                          lut16 (fp16[16]); p1 = packed zeros (fp16) or packed
 *                          absmax (fp32).  W2/W4/W8 give s*(q-z) (exact in fp32);
 *                          LUT4 gives fp32(lut[q]) * absmax rounded to nearest.
 * ------------------------------------------------------------------------- */
ql_status qlinear_debug_unpack(int fmt, const void* packed, uint8_t* codes, int N, int K,
                               ql_stream_t stream);
ql_status qlinear_debug_dequant(int fmt, const void* packed, const void* p0, const void* p1,
                                float* w, int N, int K, ql_stream_t stream);

/* ---------------------------------------------------------------------------
 * Launch plan (host, for tuning and reporting): CTAs, warps per CTA and work units of
 * the GEMV launch that a call with these arguments would make on the current device.
 * ------------------------------------------------------------------------- */
typedef struct {
  int ctas;         /* persistent CTAs launched */
  int warps;        /* warps per CTA */
  int tiles_per_warp;
  long long units;  /* (128-column block, 128-element group) work units */
  int m_bucket;     /* 1: M <= 8, 2: M <= 16 */
  int warps_per_unit; /* consumer warps that share one work unit (1, 2 or 4) */
} ql_plan;

ql_status qlinear_plan(int fmt, int M, int N, int K, ql_plan* plan);

#ifdef __cplusplus
}
#endif
#endif /* QLINEAR_H_ */
