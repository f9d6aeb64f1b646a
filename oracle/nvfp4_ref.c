/*
 * nvfp4_ref.c -- CPU oracle for NVFP4 block quantization with ScaleSearch.
 *
 * TEST INFRASTRUCTURE ONLY: the plain definition the CUDA library is checked against.
 * Single-threaded C99, IEEE binary32 with round-to-nearest-even, built with -ffp-contract=off and
 * without fast-math, subnormals kept.  Number-format converters are integer bit manipulation;
 * no hardware FP8/FP4 conversion is used.  Shares nothing with the CUDA path.
 *
 * Page citations are by page title and section (see nvfp4_ref.h for the page list).
 */
#include "nvfp4_ref.h"

#include <float.h>
#include <math.h>
#include <string.h>

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

static float qnan(void) { return u2f(0x7FC00000u); }
static float pow2f(int k);

/* Nearest integer to a non-negative finite w < 2^24, ties to even, from w's bits. */
static uint32_t rne_int(float w) {
  uint32_t b = f2u(w);
  uint32_t e = (b >> 23) & 0xFFu;
  if (e < 126u) return 0u; /* w < 0.5 */
  uint32_t s = (b & 0x7FFFFFu) | 0x800000u; /* w = s * 2^(e-150) */
  if (e >= 150u) return s << (e - 150u);
  uint32_t sh = 150u - e; /* 1..24 fraction bits */
  uint32_t ip = s >> sh;
  uint32_t rem = s & ((1u << sh) - 1u);
  uint32_t half = 1u << (sh - 1u);
  if (rem > half || (rem == half && (ip & 1u))) ip += 1u;
  return ip;
}

/* ---------------------------------------------------------------------------------------------
 * E2M1: 1 sign, 2 exponent, 1 mantissa bit ([E2M1] page, "FP4 の仕組みと利点"; [NVFP4] page,
 * "超低精度推論を支えるアーキテクチャ").  With exponent bias 1 the magnitudes are
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}; 6 is the largest, which is the divisor of max-scaling on the
 * ScaleSearch page (s = round(amax / 6)).
 * ------------------------------------------------------------------------------------------- */
float ref_e2m1_decode(uint8_t code) {
  int e = (code >> 1) & 3, m = code & 1;
  float v = (e == 0) ? 0.5f * (float)m                      /* subnormal: m * 2^(1-bias) / 2 */
                     : ldexpf(1.0f + 0.5f * (float)m, e - 1); /* (1 + m/2) * 2^(e - bias) */
  return (code & 8) ? -v : v;
}

uint8_t ref_e2m1_encode(float y) {
  uint8_t sign = (f2u(y) >> 31) ? 0x8 : 0x0;
  float a = fabsf(y);
  uint8_t mag;
  if (!(a < 6.0f)) {
    mag = 7; /* |y| >= 6 saturates to 6 (finite inputs only) */
  } else if (a < 2.0f) {
    mag = (uint8_t)rne_int(a * 2.0f); /* spacing 0.5 on [0,2): codes 0..4 */
  } else if (a < 4.0f) {
    mag = (uint8_t)(rne_int(a) + 2u); /* spacing 1 on [2,4): 2,3,4 -> codes 4,5,6 */
  } else {
    mag = (uint8_t)(rne_int(a * 0.5f) + 4u); /* spacing 2 on [4,6): 4,6 -> codes 6,7 */
  }
  return (uint8_t)(sign | mag);
}

/* ---------------------------------------------------------------------------------------------
 * E4M3 (the "fn" FP8 variant): bias 7, no infinities, exponent 15 with mantissa 7 is NaN, so the
 * largest finite value is 1.75 * 2^8 = 448 (the FP8 maximum used on the BEVFormer page, section 7).
 * The ScaleSearch page calls the block scale "UE4M3": the unsigned use of the same 8-bit code.
 * ------------------------------------------------------------------------------------------- */
float ref_e4m3_decode(uint8_t code) {
  int e = (code >> 3) & 0xF, m = code & 7;
  float v;
  if (e == 15 && m == 7) v = qnan();
  else if (e == 0) v = ldexpf((float)m, -9);        /* subnormal: m/8 * 2^(1-7) */
  else v = ldexpf((float)(8 + m), e - 10);          /* (1 + m/8) * 2^(e-7) */
  return (code & 0x80) ? -v : v;
}

uint8_t ref_e4m3_encode(float v) {
  uint8_t sign = (f2u(v) >> 31) ? 0x80 : 0x00;
  float a = fabsf(v);
  if (a != a) return (uint8_t)(sign | 0x7F);
  if (!(a < 448.0f)) return (uint8_t)(sign | 0x7E); /* saturate (also +inf) */
  uint32_t be = (f2u(a) >> 23) & 0xFFu;
  int k = (int)be - 127; /* a in [2^k, 2^(k+1)) when normal */
  if (be == 0u || k < -6) {
    /* E4M3 subnormal range: quantum 2^-9; n == 8 is the smallest normal, code 0x08 */
    uint32_t n = rne_int(ldexpf(a, 9));
    return (uint8_t)(sign | n);
  }
  uint32_t n = rne_int(ldexpf(a, 3 - k)); /* significand in units of 2^(k-3): 8..16 */
  int ee = k + 7;
  if (n == 16u) { n = 8u; ee += 1; }
  uint32_t code = ((uint32_t)ee << 3) | (n - 8u);
  if (code > 0x7Eu) code = 0x7Eu;
  return (uint8_t)(sign | code);
}

/* ---- dtype helpers ---- */
float ref_bf16_to_f32(uint16_t h) { return u2f((uint32_t)h << 16); }

float ref_f16_to_f32(uint16_t h) {
  uint32_t s = (h >> 15) & 1u, e = (h >> 10) & 0x1Fu, m = h & 0x3FFu;
  float v;
  if (e == 0u) v = ldexpf((float)m, -24);
  else if (e == 31u) v = m ? qnan() : INFINITY;
  else v = ldexpf((float)(m | 0x400u), (int)e - 25);
  return s ? -v : v;
}

uint16_t ref_f32_to_bf16(float f) {
  uint32_t b = f2u(f);
  if ((b & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((b >> 16) | 0x40u);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

uint16_t ref_f32_to_f16(float f) {
  uint16_t s = (uint16_t)((f2u(f) >> 16) & 0x8000u);
  float a = fabsf(f);
  if (a != a) return (uint16_t)(s | 0x7E00u);
  if (a >= 65520.0f) return (uint16_t)(s | 0x7C00u); /* at or past the midpoint above 65504 */
  if (a < ldexpf(1.0f, -14)) {
    uint32_t n = rne_int(ldexpf(a, 24)); /* subnormal quantum 2^-24; 1024 = smallest normal */
    return (uint16_t)(s | n);
  }
  int k = (int)((f2u(a) >> 23) & 0xFFu) - 127;
  uint32_t n = rne_int(ldexpf(a, 10 - k));
  int ee = k + 15;
  if (n == 2048u) { n = 1024u; ee += 1; }
  return (uint16_t)(s | (uint16_t)(((uint32_t)ee << 10) | (n - 1024u)));
}

static float load_elem(const void* x, int dtype, int64_t i) {
  if (dtype == REF_F32) return ((const float*)x)[i];
  if (dtype == REF_BF16) return ref_bf16_to_f32(((const uint16_t*)x)[i]);
  return ref_f16_to_f32(((const uint16_t*)x)[i]);
}

static void store_elem(void* out, int dtype, int64_t i, float v) {
  if (dtype == REF_F32) ((float*)out)[i] = v;
  else if (dtype == REF_BF16) ((uint16_t*)out)[i] = ref_f32_to_bf16(v);
  else ((uint16_t*)out)[i] = ref_f32_to_f16(v);
}

/* ---------------------------------------------------------------------------------------------
 * Tensor amax and the FP32 per-tensor scale ([NVFP4] page: a second-level FP32 scale per tensor).
 * The per-tensor scale maps the tensor's largest magnitude onto 6 * 448, the top of the E2M1 range
 * times the top of the E4M3 range: g = amax / 2688.
 * ------------------------------------------------------------------------------------------- */
float ref_tensor_amax(const void* x, int64_t n, int dtype) {
  uint32_t m = 0u;
  for (int64_t i = 0; i < n; ++i) {
    uint32_t b = f2u(load_elem(x, dtype, i)) & 0x7FFFFFFFu;
    if (b > m) m = b;
  }
  return u2f(m);
}

float ref_global_scale(float amax) { return amax / 2688.0f; }

/* ---------------------------------------------------------------------------------------------
 * ScaleSearch for one block ([SS] page, Method > ScaleSearch):
 *   default (max-scaling) scale s = round(amax_b / 6), here relative to the tensor scale:
 *       c0 = E4M3(fl(fl(amax_b / 6) / g))                     (code in 0..126)
 *   candidate scales from the integer view of that code: c = c0 + f, f in [f_lo, f_hi];
 *       c must be a positive finite E4M3 code (1..126); zero, NaN and sign-flipped codes are skipped
 *   each candidate is scored by the block's squared error (the MSE times 16), summed in FP32 in
 *   element order; the smallest wins, ties to the smaller |f|, then the smaller f.
 * Per element, with d = fl(dec(c) * g) and r = fl(1 / d):
 *       y = fl(x * r);  q = E2M1(y);  xh = fl(dec(q) * d);  e = fl(x - xh);  sse = fl(sse + fl(e * e))
 * The scale is applied to x by multiplying with its reciprocal, as the BEVFormer page applies its
 * per-tensor scale by one multiply.
 * ------------------------------------------------------------------------------------------- */
static float candidate_sse(const float* x, float d, float r) {
  float s = 0.0f;
  for (int i = 0; i < 16; ++i) {
    float y = x[i] * r;
    float xh = ref_e2m1_decode(ref_e2m1_encode(y)) * d;
    float e = x[i] - xh;
    s = s + e * e;
  }
  return s;
}

static void encode_block(const float* x, float r, uint8_t* codes8) {
  for (int k = 0; k < 8; ++k) {
    uint8_t lo = ref_e2m1_encode(x[2 * k] * r);
    uint8_t hi = ref_e2m1_encode(x[2 * k + 1] * r);
    codes8[k] = (uint8_t)((lo & 0xF) | ((hi & 0xF) << 4)); /* element 2k in the low nibble */
  }
}

/* Blocks that carry no scale: codes keep only each element's sign (zero of that sign). */
static void zero_block(const float* x, uint8_t* codes8) {
  for (int k = 0; k < 8; ++k) {
    uint8_t lo = (f2u(x[2 * k]) >> 31) ? 0x8 : 0x0;
    uint8_t hi = (f2u(x[2 * k + 1]) >> 31) ? 0x8 : 0x0;
    codes8[k] = (uint8_t)(lo | (hi << 4));
  }
}

/* Returns 1 and the block amax when the block and g can carry a scale; 0 after writing a poisoned
 * block (non-finite element, or g NaN / infinite / negative). */
static int block_prologue(const float* x, float g, float* amax_b, uint8_t* codes8, uint8_t* scale,
                          int8_t* fstar, float* sse) {
  float m = 0.0f;
  int finite = 1;
  for (int i = 0; i < 16; ++i) {
    float a = fabsf(x[i]);
    if (!(a <= FLT_MAX)) finite = 0;
    else if (a > m) m = a;
  }
  if (!finite || !(g >= 0.0f) || !(g <= FLT_MAX)) {
    memset(codes8, 0, 8);
    *scale = 0x7F;
    if (fstar) *fstar = -128;
    if (sse) *sse = qnan();
    return 0;
  }
  *amax_b = m;
  return 1;
}

static float zero_sse(const float* x) {
  float s = 0.0f;
  for (int i = 0; i < 16; ++i) s = s + x[i] * x[i];
  return s;
}

void ref_search_block(const float* x, float g, int f_lo, int f_hi, uint8_t* codes8, uint8_t* scale,
                      int8_t* fstar, float* sse) {
  float amax_b;
  if (!block_prologue(x, g, &amax_b, codes8, scale, fstar, sse)) return;
  if (amax_b == 0.0f) {
    zero_block(x, codes8);
    *scale = 0x00;
    if (fstar) *fstar = -128;
    if (sse) *sse = 0.0f;
    return;
  }
  float t = amax_b / 6.0f;
  float sr = t / g;
  int c0 = ref_e4m3_encode(sr);

  int span = (f_lo < 0 ? -f_lo : f_lo);
  if ((f_hi < 0 ? -f_hi : f_hi) > span) span = (f_hi < 0 ? -f_hi : f_hi);
  int have = 0, bestf = 0;
  float best = 0.0f;
  for (int j = 0; j <= 2 * span; ++j) {
    int f = (j == 0) ? 0 : ((j & 1) ? -((j + 1) / 2) : (j / 2)); /* 0, -1, +1, -2, +2, ... */
    if (f < f_lo || f > f_hi) continue;
    int c = c0 + f;
    if (c < 1 || c > 126) continue;
    float d = ref_e4m3_decode((uint8_t)c) * g;
    if (d == 0.0f) continue;
    float r = 1.0f / d;
    if (!(r <= FLT_MAX)) continue;
    float s = candidate_sse(x, d, r);
    if (!have || s < best) {
      have = 1;
      best = s;
      bestf = f;
    }
  }
  if (!have) {
    zero_block(x, codes8);
    *scale = 0x00;
    if (fstar) *fstar = -128;
    if (sse) *sse = zero_sse(x);
    return;
  }
  int cs = c0 + bestf;
  float d = ref_e4m3_decode((uint8_t)cs) * g;
  encode_block(x, 1.0f / d, codes8);
  *scale = (uint8_t)cs;
  if (fstar) *fstar = (int8_t)bestf;
  if (sse) *sse = best;
}

/* Max-scaling on its own ([SS] page: the default s = round(amax / 6)); no candidate loop. */
void ref_maxscale_block(const float* x, float g, uint8_t* codes8, uint8_t* scale, float* sse) {
  float amax_b;
  if (!block_prologue(x, g, &amax_b, codes8, scale, 0, sse)) return;
  uint8_t c0 = ref_e4m3_encode((amax_b / 6.0f) / g);
  float d = (c0 == 0 || c0 > 126) ? 0.0f : ref_e4m3_decode(c0) * g;
  float r = (d == 0.0f) ? INFINITY : 1.0f / d;
  if (amax_b == 0.0f || d == 0.0f || !(r <= FLT_MAX)) {
    zero_block(x, codes8);
    *scale = 0x00;
    if (sse) *sse = (amax_b == 0.0f) ? 0.0f : zero_sse(x);
    return;
  }
  encode_block(x, r, codes8);
  *scale = c0;
  if (sse) {
    float s = 0.0f;
    for (int i = 0; i < 16; ++i) {
      float xh = ref_e2m1_decode(ref_e2m1_encode(x[i] * r)) * d;
      float e = x[i] - xh;
      s = s + e * e;
    }
    *sse = s;
  }
}

void ref_quantize_blocks(const void* x, int dtype, int64_t b0, int64_t b1, float g, int f_lo, int f_hi,
                         uint8_t* codes, uint8_t* scales, int8_t* block_f, float* block_sse) {
  float blk[16];
  for (int64_t b = b0; b < b1; ++b) {
    for (int i = 0; i < 16; ++i) blk[i] = load_elem(x, dtype, 16 * b + i);
    int64_t o = b - b0;
    ref_search_block(blk, g, f_lo, f_hi, codes + 8 * o, scales + o, block_f ? block_f + o : 0,
                     block_sse ? block_sse + o : 0);
  }
}

int ref_quantize(const void* x, int64_t n, int dtype, int f_lo, int f_hi, const float* gscale_in,
                 uint8_t* codes, uint8_t* scales, float* gscale_out, int8_t* block_f, float* block_sse) {
  if (n < 0 || n % 16 != 0) return -2;
  float g = gscale_in ? *gscale_in : ref_global_scale(ref_tensor_amax(x, n, dtype));
  if (gscale_out) *gscale_out = g;
  ref_quantize_blocks(x, dtype, 0, n / 16, g, f_lo, f_hi, codes, scales, block_f, block_sse);
  return 0;
}

/* Dequantize: the block scale is multiplied back once ([BEV] page, section 7) and the E4M3 block
 * scale times the FP32 tensor scale gives the block's step ([NVFP4] page). */
int ref_dequantize(const uint8_t* codes, const uint8_t* scales, float g, int64_t n, int out_dtype, void* out) {
  if (n < 0 || n % 16 != 0) return -2;
  for (int64_t b = 0; b < n / 16; ++b) {
    float d = ref_e4m3_decode(scales[b]) * g;
    for (int i = 0; i < 16; ++i) {
      uint8_t byte = codes[8 * b + i / 2];
      uint8_t q = (i & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
      store_elem(out, out_dtype, 16 * b + i, ref_e2m1_decode(q) * d);
    }
  }
  return 0;
}

/* ---------------------------------------------------------------------------------------------
 * Hadamard rotation ([SS] page, ScaleSearchAttention > incoherence processing: a Hadamard
 * transform on Q and K).  Sylvester H16 in natural order, normalised by 1/4 = 1/sqrt(16), applied
 * as butterflies with strides 1, 2, 4, 8, each pair (a, b) -> (a + b, a - b), then times 0.25.
 * ------------------------------------------------------------------------------------------- */
void ref_fwht16_f32(float* a) {
  for (int h = 1; h < 16; h <<= 1) {
    for (int i = 0; i < 16; ++i) {
      if ((i & h) == 0) {
        float u = a[i], v = a[i + h];
        a[i] = u + v;
        a[i + h] = u - v;
      }
    }
  }
  for (int i = 0; i < 16; ++i) a[i] = a[i] * 0.25f;
}

int ref_hadamard16(const void* x, int64_t n, int dtype, void* out, int out_dtype) {
  if (n < 0 || n % 16 != 0) return -2;
  float blk[16];
  for (int64_t b = 0; b < n / 16; ++b) {
    for (int i = 0; i < 16; ++i) blk[i] = load_elem(x, dtype, 16 * b + i);
    ref_fwht16_f32(blk);
    for (int i = 0; i < 16; ++i) store_elem(out, out_dtype, 16 * b + i, blk[i]);
  }
  return 0;
}

/* Hadamard-16 with a random sign diagonal D (QuIP#-style incoherence processing, as cited on the
 * ScaleSearchAttention page): forward out = (H16 / 4) D x, inverse (the transpose) out = D (H16 / 4) x.
 * Bit i of `signs` set means element i of every group is negated; negation is exact.  signs = 0 and
 * either direction give ref_hadamard16. */
int ref_hadamard16_ex(const void* x, int64_t n, int dtype, void* out, int out_dtype, uint32_t signs, int inverse) {
  if (n < 0 || n % 16 != 0 || signs > 0xFFFFu) return -2;
  float blk[16];
  for (int64_t b = 0; b < n / 16; ++b) {
    for (int i = 0; i < 16; ++i) blk[i] = load_elem(x, dtype, 16 * b + i);
    if (!inverse)
      for (int i = 0; i < 16; ++i) if ((signs >> i) & 1u) blk[i] = -blk[i];
    ref_fwht16_f32(blk);
    if (inverse)
      for (int i = 0; i < 16; ++i) if ((signs >> i) & 1u) blk[i] = -blk[i];
    for (int i = 0; i < 16; ++i) store_elem(out, out_dtype, 16 * b + i, blk[i]);
  }
  return 0;
}

/* ---------------------------------------------------------------------------------------------
 * Attention-sink mixed-precision KV layout ([SS] page, ScaleSearchAttention > attention-sink-aware
 * mixed-precision caching): the first and last blocks of the cache stay at full precision, the
 * middle blocks are stored as NVFP4.  Read here as: the first `sink` and last `recent` tokens of
 * every (batch, head) row are copied verbatim (BF16), the middle tokens are optionally rotated
 * (FWHT-16 along D, kept in FP32) and quantized along D with one tensor scale over the middle.
 * ------------------------------------------------------------------------------------------- */
static void load_row_group(const uint16_t* k, int64_t off, int rotate, float* blk) {
  for (int i = 0; i < 16; ++i) blk[i] = ref_bf16_to_f32(k[off + i]);
  if (rotate) ref_fwht16_f32(blk);
}

int ref_kv_mixed(const uint16_t* k, int64_t B, int64_t H, int64_t T, int64_t D, int sink, int recent,
                 int rotate, int f_lo, int f_hi, uint16_t* sink_out, uint16_t* recent_out,
                 uint8_t* codes, uint8_t* scales, float* gscale_out) {
  if (B < 0 || H < 0 || D <= 0 || D % 16 != 0 || sink < 0 || recent < 0 || T < (int64_t)sink + recent)
    return -2;
  int64_t Tm = T - sink - recent;
  for (int64_t bh = 0; bh < B * H; ++bh) {
    const uint16_t* row = k + bh * T * D;
    if (sink) memcpy(sink_out + bh * sink * D, row, (size_t)(sink * D) * 2);
    if (recent) memcpy(recent_out + bh * recent * D, row + (T - recent) * D, (size_t)(recent * D) * 2);
  }
  float blk[16];
  uint32_t m = 0u;
  for (int64_t bh = 0; bh < B * H; ++bh)
    for (int64_t t = 0; t < Tm; ++t)
      for (int64_t j = 0; j < D / 16; ++j) {
        load_row_group(k, (bh * T + sink + t) * D + 16 * j, rotate, blk);
        for (int i = 0; i < 16; ++i) {
          uint32_t b = f2u(blk[i]) & 0x7FFFFFFFu;
          if (b > m) m = b;
        }
      }
  float g = ref_global_scale(u2f(m));
  if (gscale_out) *gscale_out = g;
  int64_t gi = 0;
  for (int64_t bh = 0; bh < B * H; ++bh)
    for (int64_t t = 0; t < Tm; ++t)
      for (int64_t j = 0; j < D / 16; ++j, ++gi) {
        load_row_group(k, (bh * T + sink + t) * D + 16 * j, rotate, blk);
        ref_search_block(blk, g, f_lo, f_hi, codes + 8 * gi, scales + gi, 0, 0);
      }
  return 0;
}

int ref_kv_append(const uint16_t* k, int64_t BH, int64_t ld_bh, int64_t first, int64_t n, int64_t D, int rotate,
                  float g, int f_lo, int f_hi, uint8_t* codes, uint8_t* scales, int64_t cap, int64_t t0) {
  if (BH < 0 || n < 0 || D <= 0 || D % 16 != 0 || t0 < 0 || t0 + n > cap || first < 0) return -2;
  float blk[16];
  for (int64_t bh = 0; bh < BH; ++bh)
    for (int64_t t = 0; t < n; ++t)
      for (int64_t j = 0; j < D / 16; ++j) {
        const int64_t out = (bh * cap + t0 + t) * (D / 16) + j;
        load_row_group(k, bh * ld_bh + (first + t) * D + 16 * j, rotate, blk);
        ref_search_block(blk, g, f_lo, f_hi, codes + 8 * out, scales + out, 0, 0);
      }
  return 0;
}

/* ---- multi-scale deformable attention forward (see the header) ---- */
static double msda_corner(const float* value, int64_t b, int64_t key0, int64_t H, int64_t W, int64_t yy, int64_t xx,
                          int64_t nkeys, int64_t heads, int64_t ch, int64_t h, int64_t c) {
  if (yy < 0 || xx < 0 || yy >= H || xx >= W) return 0.0;
  const int64_t key = key0 + yy * W + xx;
  return (double)value[((b * nkeys + key) * heads + h) * ch + c];
}

int ref_msda_forward(const float* value, const int64_t* shapes, const int64_t* start, const float* loc, const float* w,
                     int64_t bs, int64_t nkeys, int64_t heads, int64_t ch, int64_t L, int64_t P, int64_t nq, double* out) {
  for (int64_t b = 0; b < bs; ++b)
    for (int64_t q = 0; q < nq; ++q)
      for (int64_t h = 0; h < heads; ++h)
        for (int64_t c = 0; c < ch; ++c) {
          double acc = 0.0;
          for (int64_t l = 0; l < L; ++l) {
            const int64_t H = shapes[2 * l], W = shapes[2 * l + 1];
            for (int64_t p = 0; p < P; ++p) {
              const int64_t i = (((b * nq + q) * heads + h) * L + l) * P + p;
              const double x = (double)loc[2 * i] * (double)W - 0.5, y = (double)loc[2 * i + 1] * (double)H - 0.5;
              if (!(x > -1.0 && y > -1.0 && x < (double)W && y < (double)H)) continue;
              const int64_t x0 = (int64_t)floor(x), y0 = (int64_t)floor(y);
              const double fx = x - (double)x0, fy = y - (double)y0;
              const double v = (1 - fy) * (1 - fx) * msda_corner(value, b, start[l], H, W, y0, x0, nkeys, heads, ch, h, c) +
                               (1 - fy) * fx * msda_corner(value, b, start[l], H, W, y0, x0 + 1, nkeys, heads, ch, h, c) +
                               fy * (1 - fx) * msda_corner(value, b, start[l], H, W, y0 + 1, x0, nkeys, heads, ch, h, c) +
                               fy * fx * msda_corner(value, b, start[l], H, W, y0 + 1, x0 + 1, nkeys, heads, ch, h, c);
              acc += (double)w[i] * v;
            }
          }
          out[((b * nq + q) * heads + h) * ch + c] = acc;
        }
  return 0;
}

/* ---- FP4 attention softmax (see the header) ---- */
float ref_exp_ss(float x) {
  if (x != x) return x;
  if (x < -104.0f) return 0.0f;
  const float log2e = 0x1.715476p+0f;                  /* fl(1 / ln 2) */
  const float ln2_hi = 0x1.62e4p-1f;                   /* ln 2 rounded to 16 significant bits */
  const float ln2_lo = 0x1.7f7d1cp-20f;                /* fl(ln 2 - ln2_hi) */
  const float n = rintf(x * log2e);
  const float r = fmaf(n, -ln2_lo, fmaf(n, -ln2_hi, x));  /* the first step is exact */
  float p = 0x1.a01a02p-13f;                           /* 1/7!, then Horner with fused multiply-adds */
  p = fmaf(p, r, 0x1.6c16c2p-10f);                     /* 1/6! */
  p = fmaf(p, r, 0x1.111112p-7f);                      /* 1/5! */
  p = fmaf(p, r, 0x1.555556p-5f);                      /* 1/4! */
  p = fmaf(p, r, 0x1.555556p-3f);                      /* 1/3! */
  p = fmaf(p, r, 0x1p-1f);                             /* 1/2! */
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  const int k = (int)n;
  if (k >= -126) return p * pow2f(k);
  return (p * pow2f(k + 64)) * pow2f(-64);
}

int ref_softmax_quantize(const float* s, int64_t batch, int64_t Tq, int64_t Tk, int causal, int64_t q_offset,
                         int f_lo, int f_hi, uint8_t* codes, uint8_t* scales, float* row_max, float* row_sum) {
  if (batch < 0 || Tq < 0 || Tk < 0 || Tk % 16 != 0) return -2;
  const float g = ref_global_scale(1.0f);
  float blk[16];
  for (int64_t row = 0; row < batch * Tq; ++row) {
    const int64_t q = row % Tq;
    const float* sr = s + row * Tk;
    float m = -INFINITY;
    for (int64_t k = 0; k < Tk; ++k)
      if (!causal || k <= q + q_offset) m = sr[k] > m ? sr[k] : m;
    float l = 0.0f;
    for (int64_t j = 0; j < Tk / 16; ++j) {
      for (int i = 0; i < 16; ++i) {
        const int64_t k = 16 * j + i;
        blk[i] = (!causal || k <= q + q_offset) ? ref_exp_ss(sr[k] - m) : 0.0f;
        l = l + blk[i];
      }
      const int64_t b = row * (Tk / 16) + j;
      ref_search_block(blk, g, f_lo, f_hi, codes + 8 * b, scales + b, 0, 0);
    }
    row_max[row] = m;
    row_sum[row] = l;
  }
  return 0;
}

/* ---- MXFP4 (see the header) ---- */
/* floor(log2(a)) of a finite a > 0, from its bit pattern */
static int ilog2_floor(float a) {
  const uint32_t b = f2u(a) & 0x7FFFFFFFu;
  const int e = (int)(b >> 23);
  if (e > 0) return e - 127;
  int msb = 22;                              /* subnormal: a = m * 2^-149 with m = b */
  while (!((b >> msb) & 1u)) --msb;
  return msb - 149;
}

/* 2^k exactly, k in [-149, 127] */
static float pow2f(int k) {
  return k >= -126 ? u2f((uint32_t)(k + 127) << 23) : u2f(1u << (k + 149));
}

int ref_mxfp4_quantize(const void* x, int64_t n, int dtype, uint8_t* codes, uint8_t* scales) {
  if (n < 0 || n % 32 != 0) return -2;
  for (int64_t b = 0; b < n / 32; ++b) {
    float v[32], amax = 0.0f;
    int bad = 0;
    for (int i = 0; i < 32; ++i) {
      v[i] = load_elem(x, dtype, 32 * b + i);
      const float a = fabsf(v[i]);
      if (!(a <= FLT_MAX)) bad = 1;
      else if (a > amax) amax = a;
    }
    uint8_t* c = codes + 16 * b;
    if (bad) {
      scales[b] = 0xFF;
      for (int i = 0; i < 16; ++i) c[i] = 0;
      continue;
    }
    int e = amax == 0.0f ? -127 : ilog2_floor(amax) - 2;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    scales[b] = (uint8_t)(e + 127);
    const float inv = pow2f(-e);             /* x / 2^e as an exact multiply (RNE if subnormal) */
    for (int i = 0; i < 16; ++i) {
      const uint8_t lo = ref_e2m1_encode(v[2 * i] * inv), hi = ref_e2m1_encode(v[2 * i + 1] * inv);
      c[i] = (uint8_t)(lo | (hi << 4));
    }
  }
  return 0;
}

int ref_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t n, int out_dtype, void* out) {
  if (n < 0 || n % 32 != 0) return -2;
  for (int64_t b = 0; b < n / 32; ++b) {
    const float X = scales[b] == 0xFF ? qnan() : pow2f((int)scales[b] - 127);
    for (int i = 0; i < 32; ++i) {
      const uint8_t q = (uint8_t)((codes[16 * b + i / 2] >> (4 * (i & 1))) & 15u);
      store_elem(out, out_dtype, 32 * b + i, ref_e2m1_decode(q) * X);
    }
  }
  return 0;
}

/* ---- array forms of the scalar converters (plain loops; used by the converter sweeps) ---- */
void ref_e2m1_encode_n(const float* y, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = ref_e2m1_encode(y[i]);
}
void ref_e4m3_encode_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = ref_e4m3_encode(v[i]);
}
void ref_f32_to_bf16_n(const float* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = ref_f32_to_bf16(v[i]);
}
void ref_f32_to_f16_n(const float* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = ref_f32_to_f16(v[i]);
}
void ref_f16_to_f32_n(const uint16_t* h, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = ref_f16_to_f32(h[i]);
}

/* ---- tensor-core consumer layout of the block scales (see the header) ---- */
int64_t ref_sf_mma_bytes(int64_t rows, int64_t bpr) {
  const int64_t row_tiles = (rows + 127) / 128, col_tiles = (bpr + 3) / 4;
  return row_tiles * col_tiles * 512;
}

int64_t ref_sf_mma_offset(int64_t r, int64_t c, int64_t bpr) {
  const int64_t col_tiles = (bpr + 3) / 4;
  const int64_t tile = (r / 128) * col_tiles + c / 4;   /* column tiles of a row tile are consecutive */
  const int64_t rr = r % 128, cc = c % 4;
  return tile * 512 + 16 * (rr % 32) + 4 * (rr / 32) + cc;
}

void ref_scales_to_mma(const uint8_t* lin, int64_t batch, int64_t rows, int64_t bpr, uint8_t* out) {
  const int64_t per = ref_sf_mma_bytes(rows, bpr);
  for (int64_t i = 0; i < batch * per; ++i) out[i] = 0;
  for (int64_t l = 0; l < batch; ++l)
    for (int64_t r = 0; r < rows; ++r)
      for (int64_t c = 0; c < bpr; ++c) out[l * per + ref_sf_mma_offset(r, c, bpr)] = lin[(l * rows + r) * bpr + c];
}
