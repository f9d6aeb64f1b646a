/*
 * nvfp4.h -- libnvfp4: NVFP4 block quantization with ScaleSearch on NVIDIA B200 (sm_100a).
 *
 * NVFP4 ("NVIDIAのFP4推論が50倍の効率を実現", introl.com, section 超低精度推論を支えるアーキテクチャ):
 * 4-bit E2M1 values (1 sign, 2 exponent, 1 mantissa bit; magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6) in
 * micro-blocks of 16 consecutive elements, one E4M3 (FP8) scale per micro-block and one FP32 scale per
 * tensor.  ScaleSearch ("Search your block floating-point scales!", gist.science summary of arXiv
 * 2605.12464, Method > ScaleSearch) replaces the max-scaling block scale s = round(amax_b / 6) by the
 * best of its integer neighbours: the E4M3 bit pattern of s is read as an integer, an offset f in
 * [f_lo, f_hi] is added, and the offset whose block squared error is smallest wins.
 *
 * Exact semantics (the library is bit-exact with this definition):
 *   g      = fl(amax / 2688)            amax = max |x_i| over the tensor (NaN / Inf propagate)
 *   c0     = E4M3_RNE_SAT(fl(fl(amax_b / 6) / g))          amax_b = max |x_i| over the block
 *   for f in [f_lo, f_hi], visiting 0, -1, +1, -2, +2, ...:
 *     c = c0 + f must be a positive finite E4M3 code (1..126); d = fl(E4M3(c) * g) != 0; r = fl(1/d) finite
 *     sse(f) = sum over i = 0..15, in order, in FP32, of fl(e_i * e_i), where
 *              y = fl(x_i * r), q = E2M1_RNE_SAT(y), e_i = fl(x_i - fl(E2M1(q) * d))
 *   f* = argmin sse (ties: smaller |f|, then smaller f); scale byte = c0 + f*;
 *   code_i = E2M1_RNE_SAT(fl(x_i * r*)), element 2k in the low nibble of byte k of its block.
 * Special blocks: all-zero -> scale 0x00, sign-only codes, f* = -128; no usable candidate -> the same
 * with sse = sum of x_i^2; a non-finite element, or g NaN / Inf / negative -> scale 0x7F (E4M3 NaN),
 * codes 0, f* = -128, sse NaN.
 *
 * Memory: every pointer argument is device memory owned by the caller unless stated otherwise; the
 * library allocates nothing and keeps no state between calls except cached device properties and the
 * launch policy set by nvfp4_search_policy (which changes no result).
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Calls enqueue
 * work and return without synchronising; outputs are valid once the stream reaches that point.
 * Overlapping calls on different streams that write the same outputs race, as with any kernel.
 * Errors: argument errors are reported synchronously as a negative status and nothing is enqueued.
 * A CUDA launch error is returned as NVFP4_ERR_CUDA.  With the environment variable NVFP4_CHECKED=1
 * the quantize / kv calls synchronise the stream and return NVFP4_ERR_NONFINITE when the tensor held a
 * NaN or Inf (the outputs are then poisoned in-band as described above).  For tests of the CUDA error
 * path, NVFP4_FAULT_INJECT=launch makes nvfp4_dequantize(_ex) request an invalid block size, which the
 * CUDA runtime rejects on the host: the call returns NVFP4_ERR_CUDA and nothing reaches the GPU.
 * Alignment: element buffers must be 16-byte aligned (32-byte aligned inputs use 256-bit loads);
 * code buffers 8-byte aligned.  Sizes are element counts and must be multiples of 16 (one block).
 * Size limits (NVFP4_ERR_SIZE otherwise, before anything is enqueued): one-dimensional counts up to
 * 2^60 elements; the products of multi-dimensional sizes must fit in int64; calls that split block
 * indices in 32 bits (tile layouts, KV, softmax) say so and take fewer than 2^32 blocks.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { NVFP4_F32 = 0, NVFP4_BF16 = 1, NVFP4_F16 = 2 } nvfp4_dtype;

enum {
  NVFP4_OK = 0,
  NVFP4_ERR_ARG = -1,       /* null pointer, bad dtype, bad offset window, block != 16 */
  NVFP4_ERR_SIZE = -2,      /* n < 0, n % 16 != 0, or a shape that does not split into blocks */
  NVFP4_ERR_ALIGN = -3,     /* a buffer is not aligned as required */
  NVFP4_ERR_CUDA = -4,      /* a CUDA call failed (launch error) */
  NVFP4_ERR_NONFINITE = -5  /* checked mode only: the input held NaN / Inf */
};

/* Human-readable name of a status code (static string). */
const char* nvfp4_status_str(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int nvfp4_version(void);

/* Launch policy of every ScaleSearch quantize (nvfp4_quantize*, the KV calls, nvfp4_quantize_mma_t).
 * A launch of n blocks whose window has at most 32 offsets takes the first shape that fits:
 *   n * G1 <= lane1_max:  G1 = 16 lanes per block (windows up to 16 offsets) or 32, one offset per lane,
 *                         each scored with the definition, the winner found by a shuffle reduction;
 *   n * G2 <= lanes_max:  G2 = 4 lanes per block with 3 offsets each (up to 12 offsets) or 8 with 4;
 *   otherwise:            a thread per block with the certified fast score.
 * The bounds count threads (blocks x lanes per block).  Wider windows always take a thread per block.
 * Every shape writes the same bytes; the choice only moves time (defaults 65536 and 393216 threads:
 * the crossovers measured on B200).  A bound >= 0 is installed, -1 keeps the current one; the previous
 * bounds are stored through old_lane1_max / old_lanes_max when those are not NULL (host pointers).
 * Process-wide, host only (no device call).  Returns NVFP4_OK, or NVFP4_ERR_ARG for a bound below -1.
 * The pages have no counterpart: it is a launch-shape choice. */
int nvfp4_search_policy(int64_t lane1_max, int64_t lanes_max, int64_t* old_lane1_max, int64_t* old_lanes_max);

/* Tensor amax (the FP32 per-tensor scale's input; NVFP4 page, second-level FP32 scale).
 * x: n elements of `dtype`.  d_amax: one device float, overwritten with max |x_i| (NaN if any x_i is
 * NaN, else Inf if any is infinite; 0 for n == 0).  n need not be a multiple of 16. */
int nvfp4_tensor_amax(const void* x, int64_t n, int dtype, float* d_amax, void* stream);

/* Per-tensor scale from an amax: *d_gscale = fl(*d_amax / 2688).  Both are one device float (they may
 * alias).  Used by sharded callers after reducing their shard amaxes with a max. */
int nvfp4_global_scale(const float* d_amax, float* d_gscale, void* stream);

/* ScaleSearch quantize ("Search your block floating-point scales!", Method > ScaleSearch).
 * x: n elements of `dtype` (n % 16 == 0), blocks of 16 along the contiguous order.
 * block: must be 16.  f_lo <= f_hi, both in [-126, 126]; {0, 0} is plain max-scaling.
 * codes: n/2 bytes; scales: n/16 bytes; gscale: one device float receiving g.
 * Work: one read pass for amax, one read pass for the search and encode. */
int nvfp4_quantize(const void* x, int64_t n, int dtype, int block, int f_lo, int f_hi,
                   uint8_t* codes, uint8_t* scales, float* gscale, void* stream);

/* Extended quantize.  gscale_in: NULL -> as nvfp4_quantize; else a device float holding g, and the
 * amax pass is skipped (sharded tensors, calibrated scales); gscale may then be NULL.
 * block_f: NULL or n/16 int8 receiving f* (-128 for blocks without a scale);
 * block_sse: NULL or n/16 floats receiving the winning block SSE (the block MSE times 16). */
int nvfp4_quantize_ex(const void* x, int64_t n, int dtype, int block, int f_lo, int f_hi,
                      const float* gscale_in, uint8_t* codes, uint8_t* scales, float* gscale,
                      int8_t* block_f, float* block_sse, void* stream);

/* Dequantize: out_i = fl(E2M1(code_i) * fl(E4M3(scale_b) * g)), rounded to out_dtype (RNE).
 * The block scale is applied back by one multiply (BEVFormer-on-B200 page, section 7).
 * codes: n/2 bytes, scales: n/16 bytes, gscale: one device float, out: n elements. */
int nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* gscale, int64_t n,
                     int out_dtype, void* out, void* stream);

/* Quantize and dequantize in one pass (a fused round trip, e.g. simulated quantization): the outputs of
 * nvfp4_quantize_ex (codes, scales, gscale; gscale_in as there) plus out = the dequantized tensor, n
 * elements of `dtype` (the input's), bit-identical to nvfp4_dequantize(codes, scales, g, n, dtype, out)
 * ("Search your block floating-point scales!", Method > ScaleSearch; NVFP4 page, the two-level scale).
 * For windows of 1, 9 or 17 offsets the search kernel writes each block's values as soon as its scale
 * is chosen, so the codes are not read back; other widths run the two passes.  out: 16-byte aligned;
 * it may be x itself (each block is read before its own values are written) but must not overlap x
 * otherwise.  Errors as nvfp4_quantize_ex, NVFP4_ERR_ARG for out == NULL with n > 0. */
int nvfp4_quantize_dequantize(const void* x, int64_t n, int dtype, int f_lo, int f_hi, const float* gscale_in,
                              uint8_t* codes, uint8_t* scales, float* gscale, void* out, void* stream);

/* nvfp4_dequantize with a bound on the launch footprint: at most ctas_per_sm CTAs of 256 threads per
 * SM (1..8; 0 = the default 8), so that the kernel can run beside another kernel that occupies most of
 * each SM -- e.g. dequantizing a finished chunk on a second stream while the search of the next chunk
 * is still running.  Outputs are identical to nvfp4_dequantize. */
int nvfp4_dequantize_ex(const uint8_t* codes, const uint8_t* scales, const float* gscale, int64_t n,
                        int out_dtype, void* out, int ctas_per_sm, void* stream);

/* Hadamard-16 rotation ("Search your block floating-point scales!", ScaleSearchAttention >
 * incoherence processing): each contiguous group of 16 elements is multiplied by the Sylvester
 * Hadamard matrix H16 / 4, computed as butterflies with strides 1, 2, 4, 8 in FP32.
 * x and out: n elements (n % 16 == 0); out may alias x only when dtype == out_dtype. */
int nvfp4_hadamard16(const void* x, int64_t n, int dtype, void* out, int out_dtype, void* stream);

/* Hadamard-16 with a sign diagonal D, the random-sign form of QuIP#-style incoherence processing that
 * the ScaleSearchAttention page cites: bit i of `signs` (0..0xFFFF) negates element i of every group
 * of 16 (exact).  inverse = 0: out = (H16/4) D x; inverse = 1: out = D (H16/4) x, the transpose, so
 * applying both returns x up to FP32 rounding.  Q and K rotated with the same signs keep their dot
 * products.  signs = 0 gives nvfp4_hadamard16.  Other arguments and errors as nvfp4_hadamard16;
 * NVFP4_ERR_ARG for signs > 0xFFFF or inverse not 0/1. */
int nvfp4_hadamard16_ex(const void* x, int64_t n, int dtype, void* out, int out_dtype, uint32_t signs,
                        int inverse, void* stream);

/* Attention-sink mixed-precision KV layout ("Search your block floating-point scales!",
 * ScaleSearchAttention > attention-sink-aware mixed-precision caching).
 * k_bf16: K[B,H,T,D] BF16, contiguous.  D % 16 == 0, T >= sink_tokens + recent_tokens.
 * sink_bf16: [B,H,sink_tokens,D] and recent_bf16: [B,H,recent_tokens,D] receive the first and last
 * tokens verbatim.  The T_mid = T - sink - recent middle tokens are rotated along D by FWHT-16 when
 * rotate != 0 (kept in FP32) and quantized along D with one tensor scale over the rotated middle:
 * codes [B,H,T_mid,D/2], scales [B,H,T_mid,D/16], gscale one device float.
 * B * H * T_mid * D / 16 must be below 2^32 (NVFP4_ERR_SIZE). */
int nvfp4_kv_mixed(const void* k_bf16, int64_t B, int64_t H, int64_t T, int64_t D, int sink_tokens,
                   int recent_tokens, int rotate, int f_lo, int f_hi, void* sink_bf16, void* recent_bf16,
                   uint8_t* codes, uint8_t* scales, float* gscale, void* stream);

/* nvfp4_kv_mixed plus the middle tokens' dequantized values in the same pass (a fused round trip):
 * mid_out receives BF16 [B,H,T-sink-recent,D], element-aligned with the codes, equal bit for bit to
 * nvfp4_dequantize(codes, scales, gscale, n_mid, NVFP4_BF16) -- the rotated values when `rotate`.
 * For windows of 1, 9 or 17 offsets the search kernel writes them as each block's scale is chosen;
 * other widths dequantize after the search.  mid_out: 16-byte aligned, required when the middle is
 * not empty (NVFP4_ERR_ARG).  Everything else as nvfp4_kv_mixed. */
int nvfp4_kv_mixed_dequantize(const void* k_bf16, int64_t B, int64_t H, int64_t T, int64_t D, int sink_tokens,
                              int recent_tokens, int rotate, int f_lo, int f_hi, void* sink_bf16, void* recent_bf16,
                              uint8_t* codes, uint8_t* scales, float* gscale, void* mid_out, void* stream);

/* ---- Multi-scale deformable attention forward on NVFP4 values ("自動運転モデル BEVFormer の NVIDIA Blackwell
 * B200 FP8/FP4 CUDAカーネル・チューニング", sections 5-7: only the value tensor is low precision; locations,
 * weights, interpolation and accumulation stay FP32) ----
 *   out[b,q,h,c] = sum_l sum_p w[b,q,h,l,p] * bilinear(value level l, head h, channel c; x * W_l - 0.5, y * H_l - 0.5)
 * (x, y) = loc[b,q,h,l,p]; corners outside the H_l x W_l map contribute zero; level l occupies keys
 * start_l = sum_{k<l} H_k W_k .. of the value tensor.
 * shapes: HOST array of L (H_l, W_l) pairs, 1 <= L <= 8, sum H_l W_l == nkeys (NVFP4_ERR_SIZE).
 * loc: [bs, nq, heads, L, P, 2] FP32, w: [bs, nq, heads, L, P] FP32, out: [bs, nq, heads, ch] FP32
 * (32-byte aligned).  ch (channels per head) must be 16, 32 or 64. */

/* Values as NVFP4 quantized along the channels: codes [bs, nkeys, heads, ch/2] (16-byte aligned),
 * scales [bs, nkeys, heads, ch/16] (E4M3 block scales), gscale the device tensor scale; the value
 * used is E2M1(code) * E4M3(scale) * g (the g multiply is applied once to each output). */
int nvfp4_msda_forward_nvfp4(const uint8_t* codes, const uint8_t* scales, const float* gscale, int64_t bs,
                             int64_t nkeys, int64_t heads, int64_t ch, const int64_t* shapes, int L, int P, int64_t nq,
                             const float* loc, const float* w, float* out, void* stream);

/* The full-precision twin: value [bs, nkeys, heads, ch] in dtype (FP32 / BF16 / F16, 16-byte aligned). */
int nvfp4_msda_forward(const void* value, int dtype, int64_t bs, int64_t nkeys, int64_t heads, int64_t ch,
                       const int64_t* shapes, int L, int P, int64_t nq, const float* loc, const float* w, float* out,
                       void* stream);

/* ---- MXFP4, the comparison format ("NVIDIAのFP4推論が50倍の効率を実現", 超低精度推論を支えるアーキテクチャ:
 * NVFP4 against simple power-of-two scaling such as MXFP4) ----
 * MXFP4 as the OCP Microscaling (MX) v1.0 specification defines it (not on the pages): blocks of 32
 * elements, one E8M0 scale X = 2^e, e = floor(log2(amax_b)) - 2 clamped to [-127, 127] (scale byte
 * e + 127; all-zero block: byte 0), elements E2M1_RNE_SAT(x / X) packed two per byte (element 2k in
 * the low nibble); a block holding NaN or Inf gets scale byte 0xFF and codes 0.
 * codes: n/2 bytes (16-byte aligned), scales: n/32 bytes, n % 32 == 0. */
int nvfp4_mxfp4_quantize(const void* x, int64_t n, int dtype, uint8_t* codes, uint8_t* scales, void* stream);
/* out_i = E2M1(code_i) * 2^(scale - 127) (exact in FP32), RNE to out_dtype; scale byte 0xFF gives NaN. */
int nvfp4_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t n, int out_dtype, void* out,
                           void* stream);

/* ---- Incremental KV cache for decode ("Search your block floating-point scales!", ScaleSearchAttention >
 * attention-sink mixed-precision caching, applied while the sequence grows) ----
 * The tensor scale is fixed at prefill; later tokens are quantized with it as they leave the BF16
 * window of recent tokens (values beyond 448 * 6 * g saturate). */

/* Tensor scale of a prefill: g = fl(amax / 2688) over the (rotated when rotate != 0) middle tokens
 * [sink_tokens, T - recent_tokens) of K[B,H,T,D] (BF16), exactly as nvfp4_kv_mixed computes it. */
int nvfp4_kv_gscale(const void* k_bf16, int64_t B, int64_t H, int64_t T, int64_t D, int sink_tokens, int recent_tokens,
                    int rotate, float* gscale, void* stream);

/* Quantize tokens [first, first + n) of every (batch, head) of the BF16 buffer k_bf16 [BH, T, D]
 * (optionally rotated by FWHT-16 along D) with the tensor scale *gscale into rows [t0, t0 + n) of an
 * NVFP4 cache with `cap` rows per (batch, head): codes [BH, cap, D/2]; scales [BH, cap, D/16] when
 * scale_layout == 0, or the tensor-core tile layout of BH matrices [cap, D] when scale_layout == 1
 * (nvfp4_sf_mma_bytes(cap, D, BH) bytes; padding bytes are not written).  Other rows are untouched.
 * Requires first + n <= T, t0 + n <= cap and BH * n * D / 16 < 2^32 (NVFP4_ERR_SIZE). */
int nvfp4_kv_append(const void* k_bf16, int64_t BH, int64_t T, int64_t first, int64_t n, int64_t D, int rotate,
                    int f_lo, int f_hi, const float* gscale, uint8_t* codes, uint8_t* scales, int64_t cap, int64_t t0,
                    int scale_layout, void* stream);

/* One KV append of a batch: the arguments of nvfp4_kv_append (same meaning, layout, alignment and size
 * rules), as a plain struct so that several appends can be passed at once. */
typedef struct nvfp4_kv_append_desc {
  const void* k_bf16;     /* BF16 rows [BH, T, D], device, 16-byte aligned */
  const float* gscale;    /* device float: this cache's tensor scale */
  uint8_t* codes;         /* [BH, cap, D/2], device, 8-byte aligned */
  uint8_t* scales;        /* [BH, cap, D/16], or the tile layout when scale_layout == 1 */
  int64_t BH, T, first, n, D, cap, t0;
  int32_t rotate, scale_layout;
} nvfp4_kv_append_desc;

#define NVFP4_KV_APPEND_BATCH_MAX 64

/* Several KV appends in one launch (e.g. the K and V groups of every layer of a decode step, each
 * flushing its window into its own cache): descs is a HOST array of `count` descriptors (read before
 * the call returns; count <= NVFP4_KV_APPEND_BATCH_MAX), all quantized with the window [f_lo, f_hi]
 * (at most 32 offsets, NVFP4_ERR_ARG otherwise).  Each item writes exactly the bytes nvfp4_kv_append
 * would; items must not write overlapping outputs.  Every descriptor is validated before anything is
 * launched (the first failing item's status is returned); items with BH == 0 or n == 0 are skipped.
 * A batch whose blocks together need more thread blocks than one grid holds (2^31 - 1 CTAs of 256
 * threads) returns NVFP4_ERR_SIZE, also before any launch.
 * The launch always takes lane groups (16 or 32 lanes per block while the batch is small, 4 or 8 with
 * several offsets each beyond nvfp4_search_policy's first bound): it is meant for decode-sized groups. */
int nvfp4_kv_append_batch(const nvfp4_kv_append_desc* descs, int count, int f_lo, int f_hi, void* stream);

/* ---- Tensor-core consumer ("Search your block floating-point scales!", ScaleSearchAttention: QK^T and
 * PV run as NVFP4 products on the tensor cores with FP32 accumulation) ----
 *
 * Scale tile layout.  The block-scaled tensor-core MMA reads block scales in NVIDIA's documented tile
 * format (PTX ISA, tcgen05 block scaling; not described on the pages): a matrix of `rows` rows with
 * `cols` / 16 blocks per row is cut into 512-byte tiles of 128 rows x 4 block columns (rows padded to a
 * multiple of 128, block columns to a multiple of 4, padding bytes zero).  Tiles are stored row tile
 * by row tile, the column tiles of one row tile consecutively; inside a tile the scale of row r and
 * block column c is byte 16 * (r mod 32) + 4 * (r div 32) + c.  A batch stores its matrices one after
 * another.  The codes keep the row-major packed layout of nvfp4_quantize. */

/* Bytes of the tile-layout scales of `batch` matrices of [rows, cols] (cols % 16 == 0); negative status
 * on invalid sizes. */
int64_t nvfp4_sf_mma_bytes(int64_t rows, int64_t cols, int64_t batch);

/* nvfp4_quantize_ex for x [batch, rows, cols] (contiguous, blocks along cols, cols % 16 == 0) with the
 * scales written in the tile layout: sf receives nvfp4_sf_mma_bytes(rows, cols, batch) bytes.
 * gscale_in / gscale as in nvfp4_quantize_ex (one tensor scale for the whole batch).
 * The whole tensor must hold fewer than 2^32 blocks (NVFP4_ERR_SIZE otherwise). */
int nvfp4_quantize_mma(const void* x, int64_t batch, int64_t rows, int64_t cols, int dtype, int f_lo, int f_hi,
                       const float* gscale_in, uint8_t* codes, uint8_t* sf, float* gscale, void* stream);

/* The transposed operand: x [batch, rows, cols] (contiguous) quantized in blocks of 16 consecutive
 * ROWS of each column (rows % 16 == 0), written as the [batch, cols, rows] matrices: codes_t
 * [batch, cols, rows/2] and sf_t the tile layout of cols-row matrices (nvfp4_sf_mma_bytes(cols, rows,
 * batch) bytes).  The same as nvfp4_quantize_mma of the transposed tensor; used for V in P V^T, where
 * the product contracts over tokens.  One tensor scale for the whole tensor. */
int nvfp4_quantize_mma_t(const void* x, int64_t batch, int64_t rows, int64_t cols, int dtype, int f_lo, int f_hi,
                         const float* gscale_in, uint8_t* codes_t, uint8_t* sf_t, float* gscale, void* stream);

/* nvfp4_kv_mixed with the middle-token scales in the tile layout: each (batch, head) is one
 * [T_mid, D] matrix, so sf receives nvfp4_sf_mma_bytes(T_mid, D, B * H) bytes; it feeds
 * nvfp4_gemm_nt as the K operand of Q K^T directly. */
int nvfp4_kv_mixed_mma(const void* k_bf16, int64_t B, int64_t H, int64_t T, int64_t D, int sink_tokens,
                       int recent_tokens, int rotate, int f_lo, int f_hi, void* sink_bf16, void* recent_bf16,
                       uint8_t* codes, uint8_t* sf, float* gscale, void* stream);

/* Batched NVFP4 product on the tensor cores:
 *   D[l][m][n] = alpha * g_a * g_b * sum_k A[l][m][k] * B[l][n][k]     (FP32 accumulation)
 * where A[l][m][k] = E2M1(a code) * E4M3(a scale) is operand A before its tensor scale (likewise B).
 * a_codes: [batch, M, K/2] packed codes (nvfp4_quantize_mma of a [batch, M, K] tensor), a_sf its tile
 * layout scales, a_gscale its device tensor scale; b_* likewise for [batch, N, K].
 * d: [batch, M, N] row-major, d_dtype NVFP4_F32 or NVFP4_BF16 (RNE from FP32).
 * alpha_work: one device float owned by the caller; it receives fl(fl(alpha * g_a) * g_b), which the
 * epilogue multiplies in, so it must not be shared with a concurrent call on another stream.
 * Requirements: K % 32 == 0 (NVFP4_ERR_SIZE); codes, scales and d 16-byte aligned and N * sizeof(d
 * element) a multiple of 16 (NVFP4_ERR_ALIGN); all sizes below 2^31.  K == 0 writes zeros.
 * A scale byte 0x7F (a poisoned block) makes the outputs that use it NaN. */
int nvfp4_gemm_nt(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gscale, const uint8_t* b_codes,
                  const uint8_t* b_sf, const float* b_gscale, int64_t batch, int64_t M, int64_t N, int64_t K,
                  float alpha, void* d, int d_dtype, float* alpha_work, void* stream);

/* nvfp4_gemm_nt for callers that cannot allocate device memory -- code running where cudaMalloc is not
 * available to it or not allowed (a host framework that owns every device allocation through its own
 * pool, a runtime that has reserved all device memory up front, code that must not allocate between
 * setup and teardown) and so cannot provide the alpha_work word.  The paper has no counterpart: this is
 * an interface choice of the library.
 * Same arguments, results and errors as nvfp4_gemm_nt, without alpha_work: the scale word lives in a
 * device array compiled into the library (one FP32 word, 256-byte aligned), present on every GPU that
 * loads the library until the process exits.  The word does not grow with the sizes, so no size is too
 * large for it; sizes are checked exactly as nvfp4_gemm_nt checks them.
 * The first call on a device looks up that array's address (cudaGetSymbolAddress, no allocation) and
 * returns NVFP4_ERR_CUDA if that fails; make that first call before any stream capture.  Nothing here
 * calls cudaMalloc or cudaFree.  Each call overwrites the word before its product reads it, so nothing
 * carries over from the previous call; but all calls on one device share the word, so two calls that can
 * run at the same time on the GPU (different streams without ordering) race on it and may use each
 * other's scale. */
int nvfp4_gemm_nt_noalloc(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gscale,
                          const uint8_t* b_codes, const uint8_t* b_sf, const float* b_gscale, int64_t batch,
                          int64_t M, int64_t N, int64_t K, float alpha, void* d, int d_dtype, void* stream);

/* Softmax numerators for the P V^T product of FP4 attention ([SS] ScaleSearchAttention; the pages do
 * not say how P is formed, this is the flash-attention form).  s: scores [batch, Tq, Tk] FP32 (16-byte
 * aligned, Tk % 16 == 0).  For each row (b, q): m = max over the allowed keys (causal != 0: key k is
 * allowed iff k <= q + q_offset), P~_k = exp(S_k - m) for allowed keys and 0 otherwise, l = sum_k P~_k.
 * exp is a fixed FP32 method: n = rint(x log2 e), r = fma(n, -ln2_lo, fma(n, -ln2_hi, x)) (ln 2 split at
 * 16 significant bits), p = degree-7 Taylor polynomial of e^r in Horner form with fused multiply-adds,
 * result p 2^n (0 below -104).
 * P~ is ScaleSearch-quantized along the keys (window [f_lo, f_hi] of 1, 9 or 17 offsets) with the tensor
 * scale g = fl(1/2688): codes [batch, Tq, Tk/2], sf the tile layout of the [Tq, Tk] matrices
 * (nvfp4_sf_mma_bytes(Tq, Tk, batch) bytes), *gscale = g, row_max / row_sum [batch * Tq] (FP32; the
 * sum's order is unspecified).  Then O = (P~ V) / l: nvfp4_gemm_nt of (codes, sf, gscale) with V from
 * nvfp4_quantize_mma_t, followed by nvfp4_rows_divide. */
int nvfp4_softmax_quantize_mma(const float* s, int64_t batch, int64_t Tq, int64_t Tk, int causal, int64_t q_offset,
                               int f_lo, int f_hi, uint8_t* codes, uint8_t* sf, float* gscale, float* row_max,
                               float* row_sum, void* stream);

/* x[r, c] = fl(x[r, c] / l[r]) for an FP32 [rows, cols] matrix (cols % 4 == 0, 16-byte aligned). */
int nvfp4_rows_divide(float* x, const float* l, int64_t rows, int64_t cols, void* stream);

/* FP4 attention with the scores kept on chip ([SS] ScaleSearchAttention > native NVFP4 execution): the
 * same result as
 *   S = nvfp4_gemm_nt(Q, K, alpha);  nvfp4_softmax_quantize_mma(S, causal, q_offset, f_lo, f_hi);
 *   O = nvfp4_gemm_nt(P~, V^T);  nvfp4_rows_divide(O, row_sum)
 * without the scores leaving the SMs.  Per head and 128 query rows, the 64-key tiles holding an allowed key
 * are cut into `splits` contiguous ranges.  Kernels run on `stream`: the first writes Q, K and V^T into the
 * workspace as FP16 tiles (exact); one forms S on the tensor cores (in tensor memory) and takes row maxima
 * over (splits + 1) / 2 ranges; one forms S again per range, the numerators exp(S - m) with m the maximum
 * over all keys, quantizes them (window [f_lo, f_hi] of 1, 9 or 17 offsets, tensor scale fl(1/2688)) and
 * accumulates P~ V^T; with splits > 1 the last adds the ranges' accumulators and row sums and divides.
 * Both products are FP32 sums of the exact products of the NVFP4 operands (the summation order differs from
 * nvfp4_gemm_nt's and depends on splits); P~'s codes are those of nvfp4_softmax_quantize_mma applied to this
 * call's scores, and row_sum adds its numerators in a fixed order: per key range and 16-key column block of
 * the 64-key tiles, the even and the odd keys in two FP32 sums tile by tile, added; the four column blocks,
 * then the ranges, added in order.
 * Operands (device, from the library's quantizers): q_codes [H, Tq, D/2] with q_sf the tile layout of the
 * H [Tq, D] matrices (nvfp4_quantize_mma / nvfp4_kv_mixed_mma) and q_gscale; k_* likewise for [H, Tk, D];
 * v_codes_t [H, D, Tk/2] with v_sf_t the tile layout of the H [D, Tk] matrices (nvfp4_quantize_mma_t).
 * Code arrays 8-byte aligned, k_sf 4-byte aligned (NVFP4_ERR_ALIGN otherwise).
 * alpha multiplies the scores (with the two tensor scales, rounded as nvfp4_gemm_nt rounds them); causal:
 * key k allowed for query q iff k <= q + q_offset.
 * splits: 1 .. 64 (nvfp4_attention_fused_splits gives the count that fills the current device; any count
 * gives a valid result).  workspace: caller-owned device memory, 16-byte aligned, at least
 * nvfp4_attention_fused_workspace_bytes(H, Tq, Tk, splits) bytes (NVFP4_ERR_SIZE otherwise); it holds Q, K
 * and V^T expanded to FP16 tiles (exact) and the ranges' row maxima, row sums and accumulators between the
 * kernels, so calls that share a workspace must be ordered on one stream.
 * Outputs: out [H, Tq, D] FP32 (16-byte aligned), row_max and row_sum [H * Tq].  Optional (NULL to skip;
 * for verification): s_out [H, Tq, Tk] FP32 scores (16-byte aligned; the 64-key tiles past the last
 * allowed key of all 128 rows of a query tile are not formed and not written), p_codes [H, Tq, Tk/2] and
 * p_sf (tile layout of the H [Tq, Tk] matrices; zero blocks on those tiles) -- both or neither; status: set
 * nonzero if a wait for the tensor cores ran out (the outputs are then not valid).
 * Sizes: D == 128, Tq % 128 == 0, Tk % 64 == 0, 0 < Tk < 2^26, H <= 65535 (NVFP4_ERR_SIZE otherwise). */
int nvfp4_attention_fused(const uint8_t* q_codes, const uint8_t* q_sf, const float* q_gscale, const uint8_t* k_codes,
                          const uint8_t* k_sf, const float* k_gscale, const uint8_t* v_codes_t, const uint8_t* v_sf_t,
                          const float* v_gscale, int64_t H, int64_t Tq, int64_t Tk, int64_t D, float alpha, int causal,
                          int64_t q_offset, int f_lo, int f_hi, int splits, void* workspace, size_t workspace_bytes,
                          float* out, float* row_max, float* row_sum, float* s_out, uint8_t* p_codes, uint8_t* p_sf,
                          int* status, void* stream);

/* The number of key ranges for nvfp4_attention_fused that fills the current device with equal waves of
 * CTAs (from its SM count and the kernel's occupancy; ranges of at least 8 tiles), into *splits.  Host only
 * (queries the device).  Sizes as nvfp4_attention_fused's (NVFP4_ERR_SIZE otherwise). */
int nvfp4_attention_fused_splits(int64_t H, int64_t Tq, int64_t Tk, int* splits);

/* Bytes of workspace nvfp4_attention_fused needs for H heads, Tq query rows, Tk keys and `splits` ranges:
 * the ranges' row maxima (4 H Tq splits bytes) and, when splits > 1, row sums and O accumulators
 * (4 H Tq splits (D + 1)), rounded up to 256, plus K, V^T and Q in FP16 ((2 Tk + Tq) H D 2 bytes); 0 for
 * invalid arguments.  Host only. */
size_t nvfp4_attention_fused_workspace_bytes(int64_t H, int64_t Tq, int64_t Tk, int splits);

/* Host only, for verification: the byte offsets at which nvfp4_gemm_nt reads the scale of (matrix l,
 * row r, block column c), for l < batch, r < rows, c < K/16 in that (row-major) order, into out
 * (batch * rows * K/16 entries).  No device work. */
int nvfp4_gemm_sf_offsets(int64_t rows, int64_t K, int64_t batch, int64_t* out);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H */
