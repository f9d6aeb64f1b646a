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

struct SoftmaxParams {
  const float* s;        // scores [rows = batch * Tq, Tk]
  int64_t rows, Tq, Tk;
  int causal;            // key k allowed for query q iff k <= q + q_offset
  int64_t q_offset;
  int v8;                // s is 32-byte aligned
  float* row_max;        // [rows]
  float* row_sum;        // [rows]
  float* gscale_out;     // receives g (one float), for the product that consumes P
};

// The numerators of block j of a row from its 16 scores x: minus the row maximum, through exp; masked
// keys (beyond lim) 0.
__device__ __forceinline__ void softmax_numerators(int64_t j, float m, int64_t lim, float (&x)[16]) {
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    float ea = __fsub_rn(x[i], m), eb = __fsub_rn(x[i + 1], m);
    exp_ss2(ea, eb);
    x[i] = ea;
    x[i + 1] = eb;
  }
  if (16 * j + 15 > lim) {   // the block reaches past the last allowed key
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (16 * j + i > lim) x[i] = 0.0f;
  }
}

__device__ __forceinline__ void softmax_block(const float* sr, int64_t j, float m, int64_t lim, bool v8, float (&x)[16]) {
  load_block<DT_F32>(reinterpret_cast<const char*>(sr + 16 * j), v8, x);
  softmax_numerators(j, m, lim, x);
}

// One warp per score row: pass 1 the row maximum; pass 2 the numerators of 16-key blocks (32 blocks per
// warp-uniform round, one per lane), their sum, and each block's ScaleSearch quantization.  Blocks the
// certified fast score cannot decide are queued per warp and scored with the definition 32 at a time
// (one per lane) at the end of the row, so a rare block does not hold up its warp.
constexpr int kSoftmaxDeferCap = 64;

template <int NC>
__global__ void __launch_bounds__(256) softmax_quantize_kernel(QuantParams p, SoftmaxParams a) {
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
  const int lane = threadIdx.x & 31;
  const unsigned lanes_below = (1u << lane) - 1u;
  int* dlist = defer[threadIdx.x >> 5];
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t bpr = a.Tk / 16;
  const bool v8 = a.v8 != 0;
  for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < a.rows; row += nwarps) {
    const int64_t q = row % a.Tq;
    const int64_t lim = a.causal ? q + a.q_offset : a.Tk - 1;   // last allowed key
    const float* sr = a.s + row * a.Tk;
    float m = -INFINITY;
    for (int64_t k = 4 * (int64_t)lane; k < a.Tk; k += 128) {
      const float4 v = *reinterpret_cast<const float4*>(sr + k);
      if (k <= lim) m = fmaxf(m, v.x);
      if (k + 1 <= lim) m = fmaxf(m, v.y);
      if (k + 2 <= lim) m = fmaxf(m, v.z);
      if (k + 3 <= lim) m = fmaxf(m, v.w);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
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
    for (int64_t j0 = 0; j0 < bpr; j0 += 32) {   // warp-uniform rounds
      const int64_t j = j0 + lane;
      bool deferred = false;
      if (j < bpr) {
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
    if (lane == 0) {
      a.row_max[row] = m;
      a.row_sum[row] = l;
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
