// attention.cuh -- the FP4-attention softmax: quantized softmax numerators for the P V^T product.
//
// "Search your block floating-point scales!" (gist.science summary of arXiv 2605.12464),
// ScaleSearchAttention: QK^T and PV run in NVFP4 on the tensor cores with FP32 accumulation.  For the
// PV product the softmax numerators are quantized: for each score row (batch, query) over the keys,
//   m = max over the allowed keys,  P~_k = exp(S_k - m) (allowed) or 0 (masked),  l = sum_k P~_k,
// and P~ is ScaleSearch-quantized along the keys with the tensor scale g = fl(1 / 2688) (every row's
// maximum numerator is exactly exp(0) = 1).  The output O = (P~_q V) / l then needs only a row divide.
// exp is computed by a published method in a fixed FP32 order (Cody-Waite reduction with ln 2 split at
// 16 significant bits, degree-7 Taylor polynomial in Horner form with fused multiply-adds, exact
// power-of-two scaling), so its results are reproducible bit for bit.
#pragma once

#include "search.cuh"

namespace nvfp4 {

// exp(x) of a pair: x < -104 -> 0, NaN -> NaN, otherwise p(r) * 2^n as described above, with
// n = rint(x log2 e), r = fma(n, -ln2_lo, fma(n, -ln2_hi, x)) (the inner step exact) and the Horner steps
// as fused multiply-adds; each lane of the packed FP32x2 operations rounds exactly like the scalar form.
__device__ __forceinline__ float exp_scale(float p, float n, float x) {
  if (x != x) return x;
  if (x < -104.0f) return 0.0f;
  const int k = (int)n;
  return k >= -126 ? __fmul_rn(p, pow2_exact(k)) : __fmul_rn(__fmul_rn(p, pow2_exact(k + 64)), pow2_exact(-64));
}

__device__ __forceinline__ void exp_ss2(float& a, float& b) {
  const float na = rintf(__fmul_rn(a, 0x1.715476p+0f)), nb = rintf(__fmul_rn(b, 0x1.715476p+0f));  // log2(e)
  const u64 n2 = pk2(na, nb);
  u64 r2 = fma2(n2, pk2(-0x1.62e4p-1f, -0x1.62e4p-1f), pk2(a, b));       // ln 2, high 16 bits: exact
  r2 = fma2(n2, pk2(-0x1.7f7d1cp-20f, -0x1.7f7d1cp-20f), r2);          // ln 2, remainder
  u64 p2 = pk2(0x1.a01a02p-13f, 0x1.a01a02p-13f);                      // 1/7!
  p2 = fma2(p2, r2, pk2(0x1.6c16c2p-10f, 0x1.6c16c2p-10f));             // 1/6!
  p2 = fma2(p2, r2, pk2(0x1.111112p-7f, 0x1.111112p-7f));               // 1/5!
  p2 = fma2(p2, r2, pk2(0x1.555556p-5f, 0x1.555556p-5f));               // 1/4!
  p2 = fma2(p2, r2, pk2(0x1.555556p-3f, 0x1.555556p-3f));               // 1/3!
  p2 = fma2(p2, r2, pk2(0.5f, 0.5f));                                   // 1/2!
  p2 = fma2(p2, r2, pk2(1.0f, 1.0f));
  p2 = fma2(p2, r2, pk2(1.0f, 1.0f));
  float pa, pb;
  upk2(p2, pa, pb);
  a = exp_scale(pa, na, a);
  b = exp_scale(pb, nb, b);
}

// The same exp on the 16 numerators of a block, x <- exp(x - m), with two shortcuts that leave every
// result in the range k = rint(fl((x - m) log2 e)) in [-125, 0] bit-identical:
//  * rounding: t = fl(y + 1.5 * 2^23) holds magic + rint(y) exactly (ties to even) for |y| < 2^22, so
//    n = t - magic needs no conversion instruction, and the low bits of t are k in two's complement;
//  * scaling: p lies in [2^-1, 2^1), so p * 2^k is normal for k >= -125 and its bits are bits(p) +
//    k * 2^23, i.e. bits(p) + (bits(t) << 23) (the high bits of bits(t) shift out).
// Returns false when some element is outside that range (below 2^-125, x - m < -104, NaN, or t beyond
// 2^22); the caller then recomputes the block with exp_ss2.  Elements with x - m > 0 occur only at masked
// keys, whose results are discarded.
constexpr float kRoundMagic = 0x1.8p23f;

__device__ __forceinline__ bool exp_fast16(float m, float (&x)[16]) {
  const u64 neg_m = pk2(-m, -m);   // x + (-m) rounds exactly as x - m
  const float t_min = kRoundMagic - 125.0f;
  bool ok = true;
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const u64 d2 = add2(pk2(x[i], x[i + 1]), neg_m);
    const u64 t2 = add2(mul2(d2, pk2(0x1.715476p+0f, 0x1.715476p+0f)), pk2(kRoundMagic, kRoundMagic));
    const u64 n2 = add2(t2, pk2(-kRoundMagic, -kRoundMagic));
    u64 r2 = fma2(n2, pk2(-0x1.62e4p-1f, -0x1.62e4p-1f), d2);
    r2 = fma2(n2, pk2(-0x1.7f7d1cp-20f, -0x1.7f7d1cp-20f), r2);
    u64 p2 = pk2(0x1.a01a02p-13f, 0x1.a01a02p-13f);
    p2 = fma2(p2, r2, pk2(0x1.6c16c2p-10f, 0x1.6c16c2p-10f));
    p2 = fma2(p2, r2, pk2(0x1.111112p-7f, 0x1.111112p-7f));
    p2 = fma2(p2, r2, pk2(0x1.555556p-5f, 0x1.555556p-5f));
    p2 = fma2(p2, r2, pk2(0x1.555556p-3f, 0x1.555556p-3f));
    p2 = fma2(p2, r2, pk2(0.5f, 0.5f));
    p2 = fma2(p2, r2, pk2(1.0f, 1.0f));
    p2 = fma2(p2, r2, pk2(1.0f, 1.0f));
    float pa, pb, ta, tb;
    upk2(p2, pa, pb);
    upk2(t2, ta, tb);
    ok = ok && ta >= t_min && tb >= t_min;
    // unsigned: the shift discards bits(t)'s high bits and the add wraps, both defined (a signed shift
    // that overflows is undefined behaviour)
    x[i] = __uint_as_float(__float_as_uint(pa) + (__float_as_uint(ta) << 23));
    x[i + 1] = __uint_as_float(__float_as_uint(pb) + (__float_as_uint(tb) << 23));
  }
  return ok;
}

struct SoftmaxParams {
  const float* s;        // scores [rows = batch * Tq, Tk]
  int64_t rows, Tq, Tk;
  int causal;            // key k allowed for query q iff k <= q + q_offset
  int64_t q_offset;
  int v8;                // s is 32-byte aligned
  int wpr;               // warps per row: 1, 2, 4 or 8
  float* row_max;        // [rows]
  float* row_sum;        // [rows]
  float* gscale_out;     // receives g (one float), for the product that consumes P
};

// The numerators of block j of a row from its 16 scores: minus the row maximum, through exp; masked
// keys (beyond lim) 0.  The fast exp covers every result of normal size; a block with an element outside
// its range is reloaded and computed by the general form.
__device__ __forceinline__ void softmax_block(const float* sr, int64_t j, float m, int64_t lim, bool v8, float (&x)[16]) {
  const char* src = reinterpret_cast<const char*>(sr + 16 * j);
  load_block<DT_F32>(src, v8, x);
  if (!exp_fast16(m, x)) {
    load_block<DT_F32>(src, v8, x);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      float ea = __fsub_rn(x[i], m), eb = __fsub_rn(x[i + 1], m);
      exp_ss2(ea, eb);
      x[i] = ea;
      x[i + 1] = eb;
    }
  }
  if (16 * j + 15 > lim) {   // the block reaches past the last allowed key
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (16 * j + i > lim) x[i] = 0.0f;
  }
}

// The maximum over the allowed keys among [k0, k1) of a row (k0, k1 multiples of 16), warp-reduced.
// Eight 16-byte loads per lane are issued before any is used, so a warp spends this pass waiting for
// one round trip per 4 KB rather than per 512 bytes.
__device__ __forceinline__ float row_max4(float m, const float4& v, int64_t k, int64_t lim) {
  if (k + 3 <= lim) return fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
  if (k <= lim) m = fmaxf(m, v.x);
  if (k + 1 <= lim) m = fmaxf(m, v.y);
  if (k + 2 <= lim) m = fmaxf(m, v.z);
  return m;
}

// One past the last key of the 16-key block that holds key lim (0 when no key is allowed): keys from
// there on are masked, so the maximum pass need not read them.
__device__ __forceinline__ int64_t allowed_end(int64_t lim) { return lim < 0 ? 0 : (lim & ~(int64_t)15) + 16; }

__device__ __forceinline__ float softmax_row_max(const float* sr, int64_t k0, int64_t k1, int64_t lim, int lane) {
  float m = -INFINITY;
  int64_t k = k0 + 4 * (int64_t)lane;
  for (; k + 7 * 128 < k1; k += 8 * 128) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = *reinterpret_cast<const float4*>(sr + k + 128 * u);
#pragma unroll
    for (int u = 0; u < 8; ++u) m = row_max4(m, v[u], k + 128 * u, lim);
  }
  for (; k < k1; k += 128) m = row_max4(m, *reinterpret_cast<const float4*>(sr + k), k, lim);
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  return m;
}

// Blocks [jb, je) of a row: numerators, their sum (warp-reduced, returned) and the quantization, in
// warp-uniform rounds of 32 blocks (one per lane).  Blocks the certified fast score cannot decide are
// queued per warp and scored with the definition 32 at a time (one per lane) when the queue fills and at
// the end, so a rare block does not hold up its warp.
constexpr int kSoftmaxDeferCap = 64;

template <int NC>
__device__ __forceinline__ float softmax_row_blocks(const QuantParams& p, const CandEntry* tab, const float* thr,
                                                    float inv6g, int* dlist, const float* sr, int64_t row,
                                                    int64_t bpr, int64_t jb, int64_t je, float m, int64_t lim,
                                                    bool v8, int lane) {
  const unsigned lanes_below = (1u << lane) - 1u;
  float l = 0.0f;
  int dcount = 0;  // warp-uniform
  auto flush = [&]() {
    __syncwarp();
    for (int e = lane; e < dcount; e += 32) {
      const int jd = dlist[e];
      float x[16];
      softmax_block(sr, jd, m, lim, v8, x);
      u64 x2[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) x2[k] = pk2(x[2 * k], x[2 * k + 1]);
      quantize_block_def_x2<SRC_LINEAR, false>(p, tab, thr, inv6g, false, row * bpr + jd, x2);
    }
    __syncwarp();
    dcount = 0;
  };
  for (int64_t j0 = jb; j0 < je; j0 += 32) {   // warp-uniform rounds
    const int64_t j = j0 + lane;
    bool deferred = false;
    if (j < je && 16 * j0 > lim) {
      // the whole round lies past the last allowed key: every block is zero, which quantizes to scale 0
      // and zero codes (what the full path computes for it), without exp or search
      const u64 zero[8] = {0ull, 0ull, 0ull, 0ull, 0ull, 0ull, 0ull, 0ull};
      write_block<SRC_LINEAR, false>(p, row * bpr + j, zero, TableScales{tab}, 0, -128, 0.0f, false, 0.0f);
    } else if (j < je) {
      float x[16];
      softmax_block(sr, j, m, lim, v8, x);
      u64 x2[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        l = __fadd_rn(__fadd_rn(l, x[2 * k]), x[2 * k + 1]);
        x2[k] = pk2(x[2 * k], x[2 * k + 1]);
      }
      deferred = quantize_block_fast<SRC_LINEAR, false, NC, false>(p, tab, thr, inv6g, false, row * bpr + j, x2);
    }
    if constexpr (NC > 1) {
      const unsigned msk = __ballot_sync(0xFFFFFFFFu, deferred);
      if (msk) {
        if (deferred) dlist[dcount + __popc(msk & lanes_below)] = (int)j;
        dcount += __popc(msk);
        if (dcount > kSoftmaxDeferCap - 32) flush();
      }
    }
  }
  if constexpr (NC > 1) {
    if (dcount) flush();
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) l = __fadd_rn(l, __shfl_xor_sync(0xFFFFFFFFu, l, o));
  return l;
}

// SPLIT = false: one warp per score row.  SPLIT = true (fewer, longer rows, e.g. decode): a.wpr warps per
// row (2, 4 or 8; 8 / wpr rows per CTA at a time), each over a contiguous chunk of the row's blocks; the
// chunks' maxima and sums are combined in shared memory.
template <int NC, bool SPLIT>
__global__ void __launch_bounds__(256, 4) softmax_quantize_kernel(QuantParams p, SoftmaxParams a) {
  __shared__ CandEntry tab_store[kTabSize];
  __shared__ float thr[128];
  CandEntry* tab = tab_store + kTabPad;   // indexed by code
  __shared__ int defer[8][kSoftmaxDeferCap];
  const float g = __fdiv_rn(1.0f, kTensorDiv);   // the tensor scale of numerators whose maximum is 1
  build_cand_entries(tab, g);
  build_c0_thresholds(thr, g);
  __syncthreads();
  const float inv6g = __frcp_rn(__fmul_rn(6.0f, g));
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.gscale_out = g;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int* dlist = defer[warp];
  const int64_t bpr = a.Tk / 16;
  const bool v8 = a.v8 != 0;
  if constexpr (!SPLIT) {
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < a.rows; row += nwarps) {
      const int64_t lim = a.causal ? row % a.Tq + a.q_offset : a.Tk - 1;   // last allowed key
      const float* sr = a.s + row * a.Tk;
      const float m = softmax_row_max(sr, 0, min(a.Tk, allowed_end(lim)), lim, lane);
      const float l = softmax_row_blocks<NC>(p, tab, thr, inv6g, dlist, sr, row, bpr, 0, bpr, m, lim, v8, lane);
      if (lane == 0) {
        a.row_max[row] = m;
        a.row_sum[row] = l;
      }
    }
  } else {
    __shared__ float red_max[8], red_sum[8];
    const int wpr = a.wpr, rpc = 8 / wpr;
    const int part = warp & (wpr - 1), w0 = warp & ~(wpr - 1);
    const int64_t cb = (bpr + wpr - 1) / wpr;
    const int64_t jb = min((int64_t)part * cb, bpr), je = min(jb + cb, bpr);   // this warp's blocks
    for (int64_t base = (int64_t)blockIdx.x * rpc; base < a.rows; base += (int64_t)gridDim.x * rpc) {
      const int64_t row = base + warp / wpr;   // CTA-uniform trip count: every warp reaches the barriers
      const bool live = row < a.rows;
      const int64_t lim = live && a.causal ? row % a.Tq + a.q_offset : a.Tk - 1;
      const float* sr = a.s + (live ? row : 0) * a.Tk;
      float m = live ? softmax_row_max(sr, 16 * jb, min(16 * je, allowed_end(lim)), lim, lane) : -INFINITY;
      if (lane == 0) red_max[warp] = m;
      __syncthreads();
      m = red_max[w0];
      for (int i = 1; i < wpr; ++i) m = fmaxf(m, red_max[w0 + i]);
      float l = live ? softmax_row_blocks<NC>(p, tab, thr, inv6g, dlist, sr, row, bpr, jb, je, m, lim, v8, lane) : 0.0f;
      if (lane == 0) red_sum[warp] = l;
      __syncthreads();
      if (live && part == 0 && lane == 0) {
        for (int i = 1; i < wpr; ++i) l = __fadd_rn(l, red_sum[warp + i]);
        a.row_max[row] = m;
        a.row_sum[row] = l;
      }
    }
  }
}

// x[r, c] = fl(x[r, c] / l[r]) for the [rows, cols] FP32 matrix (cols % 4 == 0, 16-byte aligned).
__global__ void __launch_bounds__(256) rows_divide_kernel(float* __restrict__ x, const float* __restrict__ l,
                                                          int64_t rows, int64_t cols) {
  const int64_t nvec = rows * cols / 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
    const float d = l[(4 * i) / cols];
    float4 v = reinterpret_cast<float4*>(x)[i];
    v.x = __fdiv_rn(v.x, d);
    v.y = __fdiv_rn(v.y, d);
    v.z = __fdiv_rn(v.z, d);
    v.w = __fdiv_rn(v.w, d);
    reinterpret_cast<float4*>(x)[i] = v;
  }
}

}  // namespace nvfp4
