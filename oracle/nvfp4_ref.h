/*
 * nvfp4_ref.h -- CPU oracle for NVFP4 block quantization with ScaleSearch.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow, single-threaded definition that the CUDA
 * library is checked against.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load it.  It shares no code, header, table or constant generator with the CUDA path.
 *
 * Sources (web pages; cited by title and section):
 *  [NVFP4]  "NVIDIAのFP4推論が50倍の効率を実現" (introl.com), section "超低精度推論を支えるアーキテクチャ":
 *           E2M1 values (1 sign, 2 exponent, 1 mantissa bit) in 16-value micro-blocks, one E4M3 FP8
 *           scale per micro-block and one FP32 scale per tensor.
 *  [E2M1]   "RTX 50 FP4" article (aitroublesolution.com), section "FP4（4ビット浮動小数点）の仕組みと利点":
 *           the 1/2/1 sign/exponent/mantissa split.
 *  [SS]     "Search your block floating-point scales!" (gist.science summary of arXiv 2605.12464),
 *           Method > ScaleSearch (mechanism, search strategy, rationale), ScaleSearchAttention
 *           (incoherence processing, attention-sink mixed-precision caching).
 *  [BEV]    "BEVFormer on B200: FP8/FP4 CUDA kernel tuning" (qiita.com), section 7 (scale applied
 *           back by one multiply; FP8 max 448; two FP4 values per uint8) and its normalised error.
 *
 * Arithmetic: IEEE binary32, round-to-nearest-even, no FMA contraction (built with
 * -ffp-contract=off, no fast-math), subnormals kept.  Converters are integer bit manipulation.
 *
 * Parity status: every function below is pinned by the not-gpu tests (library converters,
 * brute-force search, closed forms, invariants); the exact f* histogram shape on Gaussian data is
 * qualitative on the pages (bimodal) and is "parity unpinned" beyond that shape.  The block-scale tile
 * layout is pinned by an independent reshape construction of the documented tile array, hand-checked
 * offsets, padding and bijectivity; the NVFP4 product (oracle.py) by exact rational arithmetic; the
 * softmax exp (ref_exp_ss) bit for bit by the same method evaluated on exact rationals.
 */
#ifndef NVFP4_REF_H
#define NVFP4_REF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element types (same numbering as the library's dtype codes, by convention only) */
enum { REF_F32 = 0, REF_BF16 = 1, REF_F16 = 2 };

/* ---- scalar converters ---- */
/* E2M1 encode: round-to-nearest-even onto {0,.5,1,1.5,2,3,4,6}, |y|>6 saturates to 6,
 * sign bit kept (negative values that round to zero give code 0x8).  y must be finite. */
uint8_t ref_e2m1_encode(float y);
/* E2M1 decode of the low 4 bits of code. */
float ref_e2m1_decode(uint8_t code);
/* E4M3 (fn variant: bias 7, no infinities, 0x7F/0xFF = NaN) encode, RNE, saturating at 448. */
uint8_t ref_e4m3_encode(float v);
float ref_e4m3_decode(uint8_t code);
/* dtype helpers: exact widening; RNE narrowing (overflow -> inf, NaN -> quiet NaN). */
float ref_bf16_to_f32(uint16_t h);
float ref_f16_to_f32(uint16_t h);
uint16_t ref_f32_to_bf16(float f);
uint16_t ref_f32_to_f16(float f);

/* array forms (plain loops over the scalar converters) */
void ref_e2m1_encode_n(const float* y, int64_t n, uint8_t* out);
void ref_e4m3_encode_n(const float* v, int64_t n, uint8_t* out);
void ref_f32_to_bf16_n(const float* v, int64_t n, uint16_t* out);
void ref_f32_to_f16_n(const float* v, int64_t n, uint16_t* out);
void ref_f16_to_f32_n(const uint16_t* h, int64_t n, float* out);

/* ---- tensor-level steps ---- */
/* max |x_i| as the unsigned maximum of the magnitude bits: NaN/Inf propagate.  n may be 0 (-> 0). */
float ref_tensor_amax(const void* x, int64_t n, int dtype);
/* per-tensor FP32 scale g = fl(amax / (6*448)) */
float ref_global_scale(float amax);

/* One 16-element block of ScaleSearch.  x: 16 floats, g: tensor scale, offsets f in [f_lo, f_hi].
 * Outputs 8 packed code bytes (element 2k low nibble, 2k+1 high nibble), the scale byte, the chosen
 * offset (-128 when the block has no valid candidate, is all zero or is poisoned) and its SSE. */
void ref_search_block(const float* x, float g, int f_lo, int f_hi,
                      uint8_t* codes8, uint8_t* scale, int8_t* fstar, float* sse);

/* Max-scaling written on its own (no candidate loop): scale = E4M3(amax_b/6/g). */
void ref_maxscale_block(const float* x, float g, uint8_t* codes8, uint8_t* scale, float* sse);

/* Whole-tensor ScaleSearch quantize.  gscale_in: NULL -> computed from the tensor amax.
 * block_f / block_sse may be NULL.  Returns 0, or -2 if n % 16 != 0. */
int ref_quantize(const void* x, int64_t n, int dtype, int f_lo, int f_hi, const float* gscale_in,
                 uint8_t* codes, uint8_t* scales, float* gscale_out, int8_t* block_f, float* block_sse);

/* Same, over a range of blocks [b0, b1) with a given g (used for sampled full-size checks). */
void ref_quantize_blocks(const void* x, int dtype, int64_t b0, int64_t b1, float g, int f_lo, int f_hi,
                         uint8_t* codes, uint8_t* scales, int8_t* block_f, float* block_sse);

/* Dequantize: out_i = fl(dec(q_i) * fl(dec(scale_b) * g)), narrowed to out_dtype by RNE. */
int ref_dequantize(const uint8_t* codes, const uint8_t* scales, float g, int64_t n, int out_dtype, void* out);

/* 16-point fast Walsh-Hadamard transform on each contiguous group of 16, times 1/4. */
int ref_hadamard16(const void* x, int64_t n, int dtype, void* out, int out_dtype);
void ref_fwht16_f32(float* a);
/* The same with a sign diagonal D from the low 16 bits of `signs` (bit i negates element i):
 * inverse = 0: out = (H16/4) D x; inverse = 1: out = D (H16/4) x.  -2 if signs > 0xFFFF. */
int ref_hadamard16_ex(const void* x, int64_t n, int dtype, void* out, int out_dtype, uint32_t signs, int inverse);

/* Mixed-precision KV layout for K[B,H,T,D] (BF16): tokens [0,sink) and [T-recent,T) copied verbatim,
 * the rest optionally rotated (FWHT-16 along D) and ScaleSearch-quantized along D with one tensor
 * scale over the (rotated) middle tokens.  codes: [B,H,T_mid,D/2], scales: [B,H,T_mid,D/16]. */
int ref_kv_mixed(const uint16_t* k, int64_t B, int64_t H, int64_t T, int64_t D, int sink, int recent,
                 int rotate, int f_lo, int f_hi, uint16_t* sink_out, uint16_t* recent_out,
                 uint8_t* codes, uint8_t* scales, float* gscale_out);

/* Incremental KV append for decode ([SS] attention-sink mixed-precision caching, with the cache
 * growing one token group at a time): tokens [first, first+n) of every (batch, head) row block of the
 * BF16 buffer k (row block bh starts at element bh * ld_bh; token t at + t * D) are optionally
 * rotated (FWHT-16 along D) and quantized along D with the given tensor scale g (the prefill's),
 * into rows [t0, t0+n) of a cache of `cap` rows per (batch, head):
 * codes [BH, cap, D/2], scales [BH, cap, D/16] (row-major).  Other rows are left untouched.  */
int ref_kv_append(const uint16_t* k, int64_t BH, int64_t ld_bh, int64_t first, int64_t n, int64_t D, int rotate,
                  float g, int f_lo, int f_hi, uint8_t* codes, uint8_t* scales, int64_t cap, int64_t t0);

/* ---- Multi-scale deformable attention forward on quantized values ----
 * [BEV] section 5-7: only the value tensor is stored in low precision; sampling locations, attention
 * weights, the bilinear interpolation and the accumulation stay in full precision.  For every batch
 * b, query q and head h:
 *   out[b,q,h,c] = sum_l sum_p w[b,q,h,l,p] * bilinear_l(value[b, start_l + .., h, c], x * W_l - 0.5, y * H_l - 0.5)
 * with (x, y) = loc[b,q,h,l,p], level l a H_l x W_l map starting at key start_l, bilinear weights from
 * the fractional parts and corners outside the map contributing zero.  value: [bs, nkeys, heads, ch]
 * (FP32, e.g. the dequantized NVFP4 values); loc: [bs, nq, heads, L, P, 2]; w: [bs, nq, heads, L, P];
 * shapes: L pairs (H_l, W_l), start: L key offsets; out: [bs, nq, heads, ch] in double. */
int ref_msda_forward(const float* value, const int64_t* shapes, const int64_t* start, const float* loc, const float* w,
                     int64_t bs, int64_t nkeys, int64_t heads, int64_t ch, int64_t L, int64_t P, int64_t nq, double* out);

/* ---- FP4 attention: softmax numerators quantized for the P V^T product ----
 * [SS] ScaleSearchAttention runs P V^T in NVFP4 on the tensor cores.  The pages do not say how P is
 * formed; this takes the flash-attention form: for each row q of the scores S [batch, Tq, Tk],
 * m = max over the allowed keys, P~ = exp(S - m) (allowed keys) or 0 (masked keys; causal: key k is
 * allowed for query q iff k <= q + q_offset), l = sum of P~ (FP32, in key order), and P~ quantized with
 * ScaleSearch along the keys with the tensor scale g = fl(1 / 2688) (the tensor amax of P~ is 1).
 * exp is ref_exp_ss below, so both implementations produce the same P~ bit for bit. */

/* exp(x) in FP32 by Cody-Waite reduction and a degree-7 Taylor polynomial (published method, fixed
 * operation order): n = rint(x * log2(e)), r = fma(n, -ln2_lo, fma(n, -ln2_hi, x)) with ln2 split at 16
 * significant bits (the inner step is exact), p = Horner(1, 1, 1/2!, ..., 1/7!) at r with fused
 * multiply-adds, result p * 2^n (scaled in two exact steps below 2^-126).  x < -104 gives 0; NaN gives
 * NaN.  (The one place the oracle uses FMA: it is part of this method's definition.)  The pages do not
 * fix an exp; this fused form replaced an earlier one with separate multiplies and adds, and its exact
 * bits are pinned by an evaluation of the same method on exact rationals, rounded once per operation,
 * with the constants derived from ln 2 and the factorials (tests/test_oracle_attention.py). */
float ref_exp_ss(float x);

int ref_softmax_quantize(const float* s, int64_t batch, int64_t Tq, int64_t Tk, int causal, int64_t q_offset,
                         int f_lo, int f_hi, uint8_t* codes, uint8_t* scales, float* row_max, float* row_sum);

/* ---- MXFP4, the power-of-two-scaled comparison format ----
 * [NV] compares NVFP4 with "simple power-of-two scaling like MXFP4".  MXFP4 as the OCP Microscaling
 * (MX) v1.0 specification defines it: blocks of 32 elements, one E8M0 scale X = 2^e with
 * e = floor(log2(amax_b)) - 2 (2 = the exponent of E2M1's largest value 6), clamped to [-127, 127];
 * elements E2M1_RNE_SAT(x / X).  Scale byte = e + 127.  All-zero block: e = -127 (byte 0).  A block
 * with a NaN or Inf element: scale byte 0xFF (E8M0 NaN), codes 0.  Nibble order as for NVFP4.
 * codes: n/2 bytes, scales: n/32 bytes, n % 32 == 0. */
int ref_mxfp4_quantize(const void* x, int64_t n, int dtype, uint8_t* codes, uint8_t* scales);
/* x_i = E2M1(q_i) * 2^(s - 127) (exact in FP32), rounded to out_dtype; scale byte 0xFF gives NaN. */
int ref_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t n, int out_dtype, void* out);

/* ---- tensor-core consumer layout of the block scales ----
 * [SS] ScaleSearchAttention runs QK^T and PV as NVFP4 products on the tensor cores with FP32
 * accumulation.  The pages do not describe how the tensor cores read the block scales; this follows
 * NVIDIA's public description of the block-scaled MMA operands (PTX ISA, tcgen05 block scaling; cuBLAS
 * "1D block scaling factors layout"): a scale matrix of `rows` rows and `bpr` 16-element blocks per row
 * is cut into tiles of 128 rows x 4 block columns (512 bytes; rows padded to 128, columns to 4).
 * Tiles are stored row tile by row tile, the column tiles of one row tile consecutively.  Inside a
 * tile, the scale of row r and column c is byte 16 * (r mod 32) + 4 * (r div 32) + c.
 * Padding bytes are zero.  A batch of matrices stores its tiles matrix after matrix. */
int64_t ref_sf_mma_bytes(int64_t rows, int64_t bpr);                  /* one matrix, padded */
int64_t ref_sf_mma_offset(int64_t r, int64_t c, int64_t bpr);        /* byte of (row r, block c) */
/* scales in row-major [batch, rows, bpr] order -> the tile layout (out: batch * ref_sf_mma_bytes) */
void ref_scales_to_mma(const uint8_t* lin, int64_t batch, int64_t rows, int64_t bpr, uint8_t* out);

#ifdef __cplusplus
}
#endif
#endif
