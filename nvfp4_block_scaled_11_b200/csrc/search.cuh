// search.cuh -- ScaleSearch quantize for sm_100a with a certified fast score.
//
// "Search your block floating-point scales!" (gist.science summary of arXiv 2605.12464), Method >
// ScaleSearch: every offset f of the default E4M3 scale code is scored by the block's squared error and
// the best one wins.  The definition scores candidate d (r = fl(1/d)) by the in-order FP32 fold
//     F = sum_i fl(e_i^2),  e_i = fl(x_i - fl(E2M1(fl(x_i r)) d)).
// Scoring all candidates that way costs about seven FP32 operations per candidate and element.  This
// kernel scores them instead in the scaled domain,
//     P = fl(d^2) * sum_i (v_i - y_i)^2,  y_i = fl(x_i r),  v_i = E2M1(y_i),
// with the E2M1 rounding and its decode done by the hardware converters (the code never leaves an 8-bit
// register), v_i - y_i formed with one rounding by a mixed-precision subtract, and the squares
// accumulated with packed FP32 FMAs: three FP32 pipe slots per candidate and element.
//
// P differs from F only by rounding.  For blocks whose magnitudes keep every intermediate normal
// (2^-40 <= amax_b <= 2^40, every candidate d >= 2^-40, every y <= 1024) the difference is bounded by
//     |F - P| <= 2^-15 * P + 2^-15 * amax_b * Dmax + 2^-36 * amax_b^2 + 2^-140,
//     Dmax = max(d_hi, amax_b - 6 d_lo)   (d_lo / d_hi: smallest / largest candidate scale):
// both F and P are perturbations of the real sum of (x_i - v_i d)^2 by the roundings of r, y, the
// products and the sums, and |x_i - v_i d| <= d * max(1, y_max - 6) bounds the cross terms.  When the
// runner-up's score exceeds the best score by more than twice that bound, the best candidate of the
// score is the best candidate of the definition and no exact work is needed.  Otherwise the block is
// deferred and every candidate is re-scored with the definition, whose tie rule decides.  Blocks outside
// the covered range, or whose window leaves the codes 1..126 (narrow windows; wide ones score the part
// inside), are scored with the definition throughout.
#pragma once

#include "kernels.cuh"

namespace nvfp4 {

// Exact E2M1 roundings of (lo, hi), returned as the f16 halves of one register (RNE, saturating).
__device__ __forceinline__ uint32_t e2m1_round2(float lo, float hi) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %2, %1; cvt.rn.f16x2.e2m1x2 %0, t; }"
      : "=r"(r)
      : "f"(lo), "f"(hi));
  return r;
}
// E2M1 codes of 8 values packed into a word, value 2k in the low nibble of byte k.
__device__ __forceinline__ uint32_t e2m1_pack8(u64 p0, u64 p1, u64 p2, u64 p3) {
  float a0, a1, b0, b1, c0, c1, d0, d1;
  upk2(p0, a0, a1);
  upk2(p1, b0, b1);
  upk2(p2, c0, c1);
  upk2(p3, d0, d1);
  uint32_t r;
  asm("{ .reg .b8 t0, t1, t2, t3;\n"
      "  cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n"
      "  cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n"
      "  cvt.rn.satfinite.e2m1x2.f32 t2, %6, %5;\n"
      "  cvt.rn.satfinite.e2m1x2.f32 t3, %8, %7;\n"
      "  mov.b32 %0, {t0, t1, t2, t3}; }"
      : "=r"(r)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1), "f"(d0), "f"(d1));
  return r;
}
// max(m, |a|, |b|) with NaN propagation.
__device__ __forceinline__ float absmax3_nan(float m, float a, float b) {
  float d;
  asm("{ .reg .f32 u, v; abs.f32 u, %2; abs.f32 v, %3; max.NaN.f32 %0, %1, u, v; }"
      : "=f"(d)
      : "f"(m), "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ void ld_v4_b64(const void* p, u64& a, u64& b, u64& c, u64& d) {
  asm("ld.global.nc.L1::no_allocate.v4.b64 {%0,%1,%2,%3}, [%4];" : "=l"(a), "=l"(b), "=l"(c), "=l"(d) : "l"(p));
}
__device__ __forceinline__ void ld_v2_b64(const void* p, u64& a, u64& b) {
  asm("ld.global.nc.L1::no_allocate.v2.b64 {%0,%1}, [%2];" : "=l"(a), "=l"(b) : "l"(p));
}

// One 16-element block as 8 packed FP32 pairs (element 2k low, 2k+1 high).  32-byte aligned sources
// use 256-bit loads, 16-byte aligned ones 128-bit loads; 16-bit inputs are widened exactly.
template <int DT>
__device__ __forceinline__ void load_pairs(const char* src, bool v8, u64 (&x2)[8]) {
  if (DT == DT_F32) {
    if (v8) {
      ld_v4_b64(src, x2[0], x2[1], x2[2], x2[3]);
      ld_v4_b64(src + 32, x2[4], x2[5], x2[6], x2[7]);
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) ld_v2_b64(src + 16 * k, x2[2 * k], x2[2 * k + 1]);
    }
  } else {
    float x[16];
    load_block<DT>(src, v8, x);
#pragma unroll
    for (int k = 0; k < 8; ++k) x2[k] = pk2(x[2 * k], x[2 * k + 1]);
  }
}

// Candidate table for one launch, one 16-byte entry per code: d = fl(E4M3(c) * g), r = fl(1 / d) (stored
// twice so that (r, r) loads as one aligned register pair), dd = fl(d * d).  A code that cannot be a
// scale (outside 1..126, d == 0 or 1/d not finite) has r = 0 and dd = +Inf, so the fast score of such a
// candidate is 0 * Inf = NaN, whose key sorts above every finite score.  The table covers codes
// -kTabPad .. 127 + kTabPad so that a window reaching past either end of 1..126 reads only such entries.
struct __align__(16) CandEntry {
  float r, r2, dd, d;
};
constexpr int kTabPad = 16;
constexpr int kTabSize = 128 + 2 * kTabPad;

// t points at the entry of code 0 inside storage for codes -kTabPad .. 127 + kTabPad.
__device__ __forceinline__ void build_cand_entries(CandEntry* t, float g) {
  for (int i = threadIdx.x; i < kTabSize; i += blockDim.x) {
    const int c = i - kTabPad;
    const float d = c >= 0 && c <= 127 ? __fmul_rn(e4m3_value((uint32_t)c), g) : 0.0f;
    const float r = __frcp_rn(d);
    const bool ok = c >= 1 && c <= 126 && d != 0.0f && fabsf(r) <= FLT_MAX;
    const float rs = ok ? r : 0.0f;
    t[c] = CandEntry{rs, rs, ok ? __fmul_rn(d, d) : __uint_as_float(0x7F800000u), d};
  }
}

// Default code c0(a) = E4M3(fl(fl(a / 6) / g)) of a block with amax a > 0.  c0 is non-decreasing in a,
// so it is fixed by the thresholds T[k] = min{a : c0(a) >= k}: c0(a) = max{k : T[k] <= a}; T[0] = 0,
// T[127] = +Inf.  The E4M3 rounding boundary below code k is the midpoint m_k of the values of codes k-1
// and k, so T[k] lies within a few ulps of fl(fl(m_k g) 6): a short walk over neighbouring floats,
// evaluating c0 exactly as defined, stops at the float a with c0(a) >= k > c0(a - 1ulp), which is T[k]
// (the bit patterns of non-negative floats are ordered like their values).  When the estimate is not
// a positive finite float, or the walk needs more than a few steps (extreme g), bisection over the
// whole float range finds the same threshold.
__device__ __forceinline__ int c0_exact(float a, float g) {
  return a == 0.0f ? 0 : e4m3_code(__fdiv_rn(__fdiv_rn(a, 6.0f), g));
}

__device__ __forceinline__ float c0_threshold(int k, float g) {
  const float m = __fmul_rn(0.5f, __fadd_rn(e4m3_value((uint32_t)(k - 1)), e4m3_value((uint32_t)k)));
  const float a0 = __fmul_rn(__fmul_rn(m, g), 6.0f);
  if (a0 > 0.0f && a0 <= FLT_MAX) {
    uint32_t u = __float_as_uint(a0);
    for (int it = 0; it < 8; ++it) {
      if (c0_exact(__uint_as_float(u), g) >= k) {
        if (u == 0u || c0_exact(__uint_as_float(u - 1u), g) < k) return __uint_as_float(u);
        --u;
      } else {
        ++u;
      }
    }
  }
  uint32_t lo = 0u, hi = 0x7F800000u;  // c0(lo) < k <= c0(hi)
  while (hi - lo > 1u) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    if (c0_exact(__uint_as_float(mid), g) >= k) hi = mid;
    else lo = mid;
  }
  return __uint_as_float(hi);
}

__device__ __forceinline__ void build_c0_thresholds(float* T, float g) {
  for (int k = threadIdx.x; k < 128; k += blockDim.x)
    T[k] = k == 0 ? 0.0f : (k == 127 ? __uint_as_float(0x7F800000u) : c0_threshold(k, g));
}

// c0 of a finite a > 0 from the thresholds: a close first guess from one multiply, then exact steps.
__device__ __forceinline__ int c0_from_thresholds(const float* T, float a, float inv6g) {
  int c = e4m3_code(__fmul_rn(a, inv6g));
  while (T[c + 1] <= a) ++c;
  while (T[c] > a) --c;
  return c;
}

// The definition: in-order FP32 fold of the squared errors of candidate (d, r).
__device__ __forceinline__ float block_sse_def(const float (&x)[16], float d, float r) {
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float y0 = __fmul_rn(x[i], r), y1 = __fmul_rn(x[i + 1], r);
    const uint32_t h2 = e2m1_round2(y0, y1);
    const float e0 = __fsub_rn(x[i], __fmul_rn(f16lo(h2), d));
    const float e1 = __fsub_rn(x[i + 1], __fmul_rn(f16hi(h2), d));
    s = __fadd_rn(s, __fmul_rn(e0, e0));
    s = __fadd_rn(s, __fmul_rn(e1, e1));
  }
  return s;
}

__device__ __forceinline__ float block_sse_def_pairs(const u64 (&x2)[8], float d, float r) {
  float x[16];
#pragma unroll
  for (int k = 0; k < 8; ++k) upk2(x2[k], x[2 * k], x[2 * k + 1]);
  return block_sse_def(x, d, r);
}

// One element pair of the scaled-domain score: acc += (v - y)^2 for y = x * r, v = E2M1(y), both lanes.
// FIRST: acc is not read (the first pair of a candidate starts the sum with a product).
template <bool FIRST>
__device__ __forceinline__ u64 score_pair(u64 acc, u64 x2, u64 rr) {
  if (FIRST) {
    asm("{ .reg .b64 y2, e2; .reg .f32 ylo, yhi, elo, ehi; .reg .b8 q; .reg .b32 h2; .reg .b16 hl, hh;\n"
        "  mul.rn.f32x2 y2, %1, %2;\n"
        "  mov.b64 {ylo, yhi}, y2;\n"
        "  cvt.rn.satfinite.e2m1x2.f32 q, yhi, ylo;\n"
        "  cvt.rn.f16x2.e2m1x2 h2, q;\n"
        "  mov.b32 {hl, hh}, h2;\n"
        "  sub.rn.f32.f16 elo, hl, ylo;\n"
        "  sub.rn.f32.f16 ehi, hh, yhi;\n"
        "  mov.b64 e2, {elo, ehi};\n"
        "  mul.rn.f32x2 %0, e2, e2; }"
        : "=l"(acc)
        : "l"(x2), "l"(rr));
  } else {
    asm("{ .reg .b64 y2, e2; .reg .f32 ylo, yhi, elo, ehi; .reg .b8 q; .reg .b32 h2; .reg .b16 hl, hh;\n"
        "  mul.rn.f32x2 y2, %1, %2;\n"
        "  mov.b64 {ylo, yhi}, y2;\n"
        "  cvt.rn.satfinite.e2m1x2.f32 q, yhi, ylo;\n"
        "  cvt.rn.f16x2.e2m1x2 h2, q;\n"
        "  mov.b32 {hl, hh}, h2;\n"
        "  sub.rn.f32.f16 elo, hl, ylo;\n"
        "  sub.rn.f32.f16 ehi, hh, yhi;\n"
        "  mov.b64 e2, {elo, ehi};\n"
        "  fma.rn.f32x2 %0, e2, e2, %0; }"
        : "+l"(acc)
        : "l"(x2), "l"(rr));
  }
  return acc;
}

// Scaled-domain score of one candidate: sum over the block of (v - y)^2 (any order), times d^2.
__device__ __forceinline__ float score_scaled(const u64 (&x2)[8], u64 rr, float dd) {
  u64 acc = score_pair<true>(0ull, x2[0], rr);
#pragma unroll
  for (int k = 1; k < 8; ++k) acc = score_pair<false>(acc, x2[k], rr);
  float lo, hi;
  upk2(acc, lo, hi);
  return __fmul_rn(__fadd_rn(lo, hi), dd);
}


__device__ __forceinline__ bool better(float s, int f, float bs, int bf) {
  // definition order: smaller sse, then smaller |f|, then smaller f
  if (s != bs) return s < bs;
  if (abs(f) != abs(bf)) return abs(f) < abs(bf);
  return f < bf;
}

// Score every usable candidate of the window with the definition; visit 0, -1, +1, ... and keep the
// first strictly smaller SSE (the definition's tie rule).
__device__ __forceinline__ void search_def(const float (&x)[16], int c0, int f_lo, int f_hi, const CandEntry* tab,
                                           int& fstar, float& best) {
  const int span = max(abs(f_lo), abs(f_hi));
  fstar = -128;
  best = 0.0f;
  for (int jv = 0; jv <= 2 * span; ++jv) {
    const int f = (jv == 0) ? 0 : ((jv & 1) ? -((jv + 1) >> 1) : (jv >> 1));
    if (f < f_lo || f > f_hi) continue;
    const int c = c0 + f;
    if (c < 1 || c > 126) continue;
    const CandEntry e = tab[c];
    if (e.r == 0.0f) continue;
    const float s = block_sse_def(x, e.d, e.r);
    if (fstar == -128 || s < best) {
      best = s;
      fstar = f;
    }
  }
}

// Certified fast search over the NC offsets f_lo .. f_lo + NC - 1 of the default code c0.  For wide
// windows, codes outside 1..126 score NaN and never win.  Returns true with fstar / best set when the fast score
// decides the block; false when the block must be scored with the definition (outside the range the
// error bound covers, a window beyond the table or without a usable code, or a runner-up too close to
// the best).
template <int NC, bool WANT_SSE>
__device__ __forceinline__ bool search_fast(const u64 (&x2)[8], float amax_b, int c0, int f_lo,
                                            const CandEntry* tab, int& fstar, float& best) {
  const int clo = c0 + f_lo, chi = c0 + f_lo + NC - 1;
  int vlo = clo, vhi = chi;   // the codes of the window that can be scales
  if constexpr (NC >= 17) {
    // wide windows reach past 1..126 often (9.8 % of N(0,1) blocks with [-8,8]): score their valid part
    if (clo < -kTabPad || chi > 127 + kTabPad || !(amax_b >= 0x1p-40f && amax_b <= 0x1p40f)) return false;
    vlo = max(clo, 1);
    vhi = min(chi, 126);
    if (vlo > vhi) return false;
  } else {
    // narrow windows rarely do (< 2.4 %); the definition takes those, which keeps this path shorter
    if (clo < 1 || chi > 126 || !(amax_b >= 0x1p-40f && amax_b <= 0x1p40f)) return false;
  }
  const CandEntry elo = tab[vlo];
  if (elo.r == 0.0f || !(elo.d >= 0x1p-40f) || !(__fmul_rn(amax_b, elo.r) <= 1024.0f)) return false;
  const float dhi = tab[vhi].d;

  // keys: score bits with the candidate index in the low 5 bits (unsigned order = score order);
  // m1 / m2 track the smallest and the second smallest key
  uint32_t m1 = 0xFFFFFFFFu, m2 = 0xFFFFFFFFu;
#pragma unroll
  for (int j = 0; j < NC; ++j) {
    const float4 e = reinterpret_cast<const float4*>(tab)[clo + j];  // r, r, dd, d
    const float s = score_scaled(x2, pk2(e.x, e.y), e.z);
    const uint32_t key = (__float_as_uint(s) & ~31u) | (uint32_t)j;
    m2 = min(m2, max(m1, key));
    m1 = min(m1, key);
  }
  const float pbest = __uint_as_float(m1 & ~31u);
  const float p2 = __uint_as_float(m2 & ~31u);
  // bound terms (see the header): the arithmetic only has to stay an upper bound, so it uses FMAs
  const float dmax = fmaxf(dhi, __fmaf_rn(amax_b, 1.000001f, -6.0f * elo.d));
  const float beta = __fmaf_rn(amax_b, __fmaf_rn(amax_b, 0x1p-36f, dmax * 0x1p-15f), 0x1p-140f);
  const float thr = __fmaf_rn(pbest, 1.0f + 0x1p-12f, beta * 2.51f);
  if (!(p2 > thr)) return false;  // near tie: the definition decides
  fstar = f_lo + (int)(m1 & 31u);
  best = 0.0f;
  if (WANT_SSE) {
    const CandEntry e = tab[c0 + fstar];
    best = block_sse_def_pairs(x2, e.d, e.r);
  }
  return true;
}

__device__ __forceinline__ void encode_pairs(const u64 (&x2)[8], float r, uint32_t& wlo, uint32_t& whi) {
  const u64 rr = pk2(r, r);
  wlo = e2m1_pack8(mul2(x2[0], rr), mul2(x2[1], rr), mul2(x2[2], rr), mul2(x2[3], rr));
  whi = e2m1_pack8(mul2(x2[4], rr), mul2(x2[5], rr), mul2(x2[6], rr), mul2(x2[7], rr));
}

__device__ __forceinline__ float block_amax_nan(const u64 (&x2)[8]) {
  float amax_b = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float lo, hi;
    upk2(x2[k], lo, hi);
    amax_b = absmax3_nan(amax_b, lo, hi);
  }
  return amax_b;
}

template <bool ROT>
__device__ __forceinline__ void maybe_rotate(u64 (&x2)[8]) {
  if (ROT) fwht16_x2(x2);
}

// Where write_block finds the chosen scale code's r (to encode) and d (to dequantize): the launch's
// candidate table, or one lane's own candidate (d of any code computed as the table would hold it).
struct TableScales {
  const CandEntry* tab;
  __device__ __forceinline__ float r(int c) const { return tab[c].r; }
  __device__ __forceinline__ float d(int c) const { return tab[c].d; }
};
struct LaneScales {
  float rw, g;  // r of the lane's candidate (the only code it encodes with); the tensor scale
  __device__ __forceinline__ float r(int) const { return rw; }
  __device__ __forceinline__ float d(int c) const { return __fmul_rn(e4m3_value((uint32_t)c), g); }
};

// DEQ >= 0 (a dtype): also write the block's dequantized values to p.deq_out (fused round trip).
template <int MODE, bool WANT_SSE, int DEQ = -1, class SC>
__device__ __forceinline__ void write_block(const QuantParams& p, int64_t b, const u64 (&x2)[8], const SC& sc,
                                            int c0, int fstar, float sse, bool poisoned, float amax_b) {
  uint32_t wlo = 0u, whi = 0u;
  int scale;
  if (poisoned) {
    scale = 0x7F;
    sse = __uint_as_float(0x7FFFFFFFu);
  } else if (fstar != -128) {
    scale = c0 + fstar;
    encode_pairs(x2, sc.r(scale), wlo, whi);
  } else {
    // all-zero block or no usable candidate: sign-only zero codes, scale 0, sse = sum of x^2
    scale = 0;
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float lo, hi;
      upk2(x2[k], lo, hi);
      const uint32_t nib = ((__float_as_uint(lo) >> 31) << 3) | ((__float_as_uint(hi) >> 31) << 7);
      if (k < 4) wlo |= nib << (8 * k);
      else whi |= nib << (8 * (k - 4));
      if (WANT_SSE) {
        s = __fadd_rn(s, __fmul_rn(lo, lo));
        s = __fadd_rn(s, __fmul_rn(hi, hi));
      }
    }
    sse = (WANT_SSE && amax_b != 0.0f) ? s : 0.0f;
  }
  const int64_t ob = out_block<MODE>(p, b);
  reinterpret_cast<uint2*>(p.codes)[ob] = make_uint2(wlo, whi);
  p.scales[scale_index(p, ob)] = (uint8_t)scale;
  if (p.block_f) p.block_f[ob] = (int8_t)fstar;
  if (WANT_SSE) p.block_sse[ob] = sse;
  if constexpr (DEQ >= 0) {
    // d of every scale byte 0..127 is fl(E4M3(c) * g), the dequantize kernel's step
    constexpr int OS = DEQ == DT_F32 ? 4 : 2;
    store_dequantized<DEQ>(p.deq_out + 16 * OS * ob, wlo, whi, sc.d(scale), p.deq_v8 != 0);
  }
}

// Fast path for one block.  Returns true when the block needs the definition (outputs not written).
template <int MODE, bool ROT, int NC, bool WANT_SSE, int DEQ = -1>
__device__ __forceinline__ bool quantize_block_fast(const QuantParams& p, const CandEntry* tab, const float* thr,
                                                    float inv6g, bool g_bad, int64_t b, u64 (&x2)[8]) {
  maybe_rotate<ROT>(x2);
  const float amax_b = block_amax_nan(x2);
  const bool poisoned = g_bad || !(amax_b <= FLT_MAX);  // NaN / Inf element, or unusable g
  int c0 = 0, fstar = -128;
  float sse = 0.0f;
  if (!poisoned && amax_b != 0.0f) {
    c0 = c0_from_thresholds(thr, amax_b, inv6g);
    if (NC == 1) {
      const int c = c0 + p.f_lo;
      if (c >= 1 && c <= 126 && tab[c].r != 0.0f) {
        fstar = p.f_lo;
        if (WANT_SSE) sse = block_sse_def_pairs(x2, tab[c].d, tab[c].r);
      }
    } else if (!search_fast<NC, WANT_SSE>(x2, amax_b, c0, p.f_lo, tab, fstar, sse)) {
      return true;
    }
  }
  write_block<MODE, WANT_SSE, DEQ>(p, b, x2, TableScales{tab}, c0, fstar, sse, poisoned, amax_b);
  return false;
}

// The definition for one block already in registers (rotated if the path rotates): same outputs as the
// fast path, every candidate scored in order.
template <int MODE, bool WANT_SSE, int DEQ = -1>
__device__ __forceinline__ void quantize_block_def_x2(const QuantParams& p, const CandEntry* tab, const float* thr,
                                                      float inv6g, bool g_bad, int64_t b, const u64 (&x2)[8]) {
  const float amax_b = block_amax_nan(x2);
  const bool poisoned = g_bad || !(amax_b <= FLT_MAX);
  int c0 = 0, fstar = -128;
  float sse = 0.0f;
  if (!poisoned && amax_b != 0.0f) {
    c0 = c0_from_thresholds(thr, amax_b, inv6g);
    float x[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) upk2(x2[k], x[2 * k], x[2 * k + 1]);
    search_def(x, c0, p.f_lo, p.f_hi, tab, fstar, sse);
  }
  write_block<MODE, WANT_SSE, DEQ>(p, b, x2, TableScales{tab}, c0, fstar, sse, poisoned, amax_b);
}

// First element of block b (linear and KV modes: the 16 elements are contiguous).
template <int DT, int MODE>
__device__ __forceinline__ const char* block_src(const QuantParams& p, int64_t b) {
  constexpr int ES = DT == DT_F32 ? 4 : 2;
  const int64_t elem = MODE == SRC_KV ? kv_block_elem(b, p.Tm, p.bpr, p.T, p.sink, p.D) : 16 * b;
  return p.x + elem * ES;
}

// Block b as 8 packed FP32 pairs, from whichever source mode the launch uses.
template <int DT, int MODE>
__device__ __forceinline__ void load_block_pairs(const QuantParams& p, int64_t b, bool v8, u64 (&x2)[8]) {
  if constexpr (MODE == SRC_COLS) {
    constexpr int ES = DT == DT_F32 ? 4 : 2;
    uint32_t l, c, rb;
    cols_split(p, b, l, c, rb);
    float x[16];
    load_column<DT>(p.x + (((int64_t)l * p.tr_rb + rb) * 16 * p.tr_cols + c) * ES, p.tr_cols * ES, x);
#pragma unroll
    for (int k = 0; k < 8; ++k) x2[k] = pk2(x[2 * k], x[2 * k + 1]);
  } else {
    load_pairs<DT>(block_src<DT, MODE>(p, b), v8, x2);
  }
}

// The definition for one block (deferred blocks): reload, rotate, score every candidate in order.
template <int DT, int MODE, bool ROT, bool WANT_SSE, int DEQ = -1>
__device__ __forceinline__ void quantize_block_def(const QuantParams& p, const CandEntry* tab, const float* thr,
                                                   float inv6g, bool g_bad, int64_t b, bool v8) {
  u64 x2[8];
  load_block_pairs<DT, MODE>(p, b, v8, x2);
  maybe_rotate<ROT>(x2);
  quantize_block_def_x2<MODE, WANT_SSE, DEQ>(p, tab, thr, inv6g, g_bad, b, x2);
}

// One thread per 16-element block, grid-stride in warp-uniform rounds, the next block's loads in flight
// while the current one is searched.  Blocks the fast score cannot decide are queued per warp (ballot)
// and scored with the definition 32 at a time, one per lane, so a rare block does not stall its warp.
constexpr int kDeferCap = 64;
#ifndef NVFP4_SEARCH_CTAS_PER_SM
#define NVFP4_SEARCH_CTAS_PER_SM 2
#endif

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// 16-bit sources whose blocks are 32 contiguous bytes (linear tensors and the KV layout's middle tokens):
// each thread's next block is copied by cp.async into the thread's own shared-memory slot while the
// current block is searched, and widened (and rotated, when the path rotates) only when it is used.  This
// keeps the prefetched block out of registers (the register copy of a widened block costs 16 moves per
// block; measured on B200 with the C2 BF16 activations: search 130 -> 120 us, fused round trip 140 ->
// 130 us).  Two slots per thread; the two 16-byte chunks of threads 4..7 of each group of 8 are swapped
// so that a quarter-warp's 16-byte accesses fall in distinct banks.
template <int DT, int MODE, bool ROT, int NC, bool WANT_SSE, int DEQ>
__device__ __forceinline__ void search_staged(const QuantParams& p, const CandEntry* tab, const float* thr,
                                              float inv6g, bool g_bad, int64_t (*defer)[kDeferCap]) {
  static_assert(DT != DT_F32 && (MODE == SRC_LINEAR || MODE == SRC_KV), "32-byte contiguous blocks");
  __shared__ uint4 stage[2][256 * 2];
  const int t = threadIdx.x;
  const int sw = (t >> 2) & 1;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t b = (int64_t)blockIdx.x * blockDim.x + t;
  KvCursor kc;   // KV mode: the split of the block being prefetched, carried along the loop
  auto issue = [&](int64_t bb, int buf) {
    const char* src;
    if constexpr (MODE == SRC_KV) src = p.x + kc.elem(p.T, p.sink, p.D) * 2;
    else src = p.x + bb * 32;
    cp_async16((uint32_t)__cvta_generic_to_shared(&stage[buf][2 * t + sw]), src);
    cp_async16((uint32_t)__cvta_generic_to_shared(&stage[buf][2 * t + (sw ^ 1)]), src + 16);
  };
  if (b < p.nblocks) {
    if constexpr (MODE == SRC_KV) kc.init(b, stride, p.Tm, p.bpr);
    issue(b, 0);
  }
  cp_async_commit();
  const int lane = t & 31, warp = t >> 5;
  const unsigned lanes_below = (1u << lane) - 1u;
  int64_t* dlist = defer[warp];
  int dcount = 0;  // warp-uniform
  auto flush = [&]() {
    __syncwarp();
    for (int e = lane; e < dcount; e += 32)
      quantize_block_def<DT, MODE, ROT, WANT_SSE, DEQ>(p, tab, thr, inv6g, g_bad, dlist[e], p.v8 != 0);
    __syncwarp();
    dcount = 0;
  };
  int buf = 0;
  for (int64_t wb = b - lane; wb < p.nblocks; wb += stride, b += stride) {
    const bool active = b < p.nblocks;
    if (b + stride < p.nblocks) {
      if constexpr (MODE == SRC_KV) kc.advance();
      issue(b + stride, buf ^ 1);
    }
    cp_async_commit();
    cp_async_wait1();   // this thread's copy of block b has landed
    u64 x2[8];
    if (active) {
      const uint4 c0 = stage[buf][2 * t + sw], c1 = stage[buf][2 * t + (sw ^ 1)];
      const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      float x[16];
      widen_words<DT>(w, x, 8);
#pragma unroll
      for (int k = 0; k < 8; ++k) x2[k] = pk2(x[2 * k], x[2 * k + 1]);
    }
    buf ^= 1;
    const bool deferred = active && quantize_block_fast<MODE, ROT, NC, WANT_SSE, DEQ>(p, tab, thr, inv6g, g_bad, b, x2);
    if constexpr (NC > 1) {
      const unsigned m = __ballot_sync(0xFFFFFFFFu, deferred);
      if (m) {
        if (deferred) dlist[dcount + __popc(m & lanes_below)] = b;
        dcount += __popc(m);
        if (dcount > kDeferCap - 32) flush();
      }
    }
  }
  if constexpr (NC > 1) {
    if (dcount) flush();
  }
}

// 16-bit linear and KV sources take the shared-memory staged loop above; the others prefetch into registers.
template <int DT, int MODE, bool ROT>
constexpr bool kStaged = (MODE == SRC_LINEAR || MODE == SRC_KV) && DT != DT_F32;

template <int DT, int MODE, bool ROT, int NC, bool WANT_SSE, int DEQ = -1>
__global__ void __launch_bounds__(256, NVFP4_SEARCH_CTAS_PER_SM) quantize_search_kernel(QuantParams p) {
  __shared__ CandEntry tab_store[kTabSize];
  __shared__ float thr[128];
  __shared__ int64_t defer[8][kDeferCap];
  CandEntry* tab = tab_store + kTabPad;   // indexed by code
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const bool v8 = p.v8 != 0;
  int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  KvCursor kc;   // KV mode: the split of the block held in xn, carried along the loop
  auto load_next = [&](int64_t bb, u64 (&dst)[8]) {
    if constexpr (MODE == SRC_KV) {
      constexpr int ES = DT == DT_F32 ? 4 : 2;
      load_pairs<DT>(p.x + kc.elem(p.T, p.sink, p.D) * ES, v8, dst);
    } else {
      load_block_pairs<DT, MODE>(p, bb, v8, dst);
    }
  };
  u64 xn[8];
  if (!kStaged<DT, MODE, ROT> && b < p.nblocks) {
    if constexpr (MODE == SRC_KV) kc.init(b, stride, p.Tm, p.bpr);
    load_next(b, xn);  // in flight while the tables are built
  }
  float g = *p.g_src;
  if (p.g_is_amax) g = __fdiv_rn(g, kTensorDiv);
  const bool g_bad = !(g >= 0.0f) || !(g <= FLT_MAX);
  build_cand_entries(tab, g);
  if (!g_bad) build_c0_thresholds(thr, g);
  __syncthreads();
  const float inv6g = __frcp_rn(__fmul_rn(6.0f, g));
  if constexpr (kStaged<DT, MODE, ROT>) {
    search_staged<DT, MODE, ROT, NC, WANT_SSE, DEQ>(p, tab, thr, inv6g, g_bad, defer);
    return;
  }

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lanes_below = (1u << lane) - 1u;
  int64_t* dlist = defer[warp];
  int dcount = 0;  // warp-uniform
  auto flush = [&]() {
    __syncwarp();
    for (int e = lane; e < dcount; e += 32) {
      const int64_t bd = dlist[e];
      quantize_block_def<DT, MODE, ROT, WANT_SSE, DEQ>(p, tab, thr, inv6g, g_bad, bd, p.v8 != 0);
    }
    __syncwarp();
    dcount = 0;
  };

  const int64_t warp0 = b - lane;
  for (int64_t wb = warp0; wb < p.nblocks; wb += stride, b += stride) {
    const bool active = b < p.nblocks;
    u64 x2[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) x2[k] = xn[k];
    if (b + stride < p.nblocks) {
      if constexpr (MODE == SRC_KV) kc.advance();
      load_next(b + stride, xn);
    }
    const bool deferred = active && quantize_block_fast<MODE, ROT, NC, WANT_SSE, DEQ>(p, tab, thr, inv6g, g_bad, b, x2);
    if constexpr (NC > 1) {  // a single-offset window never needs the definition pass
      const unsigned m = __ballot_sync(0xFFFFFFFFu, deferred);
      if (m) {
        if (deferred) dlist[dcount + __popc(m & lanes_below)] = b;
        dcount += __popc(m);
        if (dcount > kDeferCap - 32) flush();
      }
    }
  }
  if constexpr (NC > 1) {
    if (dcount) flush();
  }
}

}  // namespace nvfp4
