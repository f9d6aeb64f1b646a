// attention.cuh -- the FP4-attention softmax: quantized softmax numerators for the P V^T product.
//
// "Search your block floating-point scales!" (gist.science summary of arXiv 2605.12464),
// ScaleSearchAttention: QK^T and PV run in NVFP4 on the tensor cores with FP32 accumulation.  For the
// PV product the softmax numerators are quantized: for each score row (batch, query) over the keys,
//   m = max over the allowed keys,  P~_k = exp(S_k - m) (allowed) or 0 (masked),  l = sum_k P~_k,
// and P~ is ScaleSearch-quantized along the keys with the tensor scale g = fl(1 / 2688) (every row's
// maximum numerator is exactly exp(0) = 1).  The output O = (P~_q V) / l then needs only a row divide.
// exp is computed by a published method in a fixed FP32 order (Cody-Waite reduction with ln 2 split at
// 16 significant bits, degree-7 Taylor polynomial in Horner form, exact power-of-two scaling), so its
// results are reproducible bit for bit.
#pragma once

#include "search.cuh"

namespace nvfp4 {

// exp(x): x < -104 -> 0, NaN -> NaN, otherwise p(r) * 2^n as described above.
__device__ __forceinline__ float exp_ss(float x) {
  if (x != x) return x;
  if (x < -104.0f) return 0.0f;
  const float n = rintf(__fmul_rn(x, 0x1.715476p+0f));                    // log2(e)
  const float r = __fsub_rn(__fsub_rn(x, __fmul_rn(n, 0x1.62e4p-1f)),    // ln 2, high 16 bits
                            __fmul_rn(n, 0x1.7f7d1cp-20f));               // ln 2, remainder
  float p = 0x1.a01a02p-13f;                                               // 1/7!
  p = __fadd_rn(__fmul_rn(p, r), 0x1.6c16c2p-10f);                         // 1/6!
  p = __fadd_rn(__fmul_rn(p, r), 0x1.111112p-7f);                          // 1/5!
  p = __fadd_rn(__fmul_rn(p, r), 0x1.555556p-5f);                          // 1/4!
  p = __fadd_rn(__fmul_rn(p, r), 0x1.555556p-3f);                          // 1/3!
  p = __fadd_rn(__fmul_rn(p, r), 0x1p-1f);                                 // 1/2!
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  const int k = (int)n;
  return k >= -126 ? __fmul_rn(p, pow2_exact(k)) : __fmul_rn(__fmul_rn(p, pow2_exact(k + 64)), pow2_exact(-64));
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

// One warp per score row: pass 1 the row maximum, pass 2 the numerators of 16-key blocks (one block per
// lane at a time), their sum, and the block's ScaleSearch quantization.  Blocks the certified fast score
// cannot decide are scored with the definition on the spot.
template <int NC>
__global__ void __launch_bounds__(256) softmax_quantize_kernel(QuantParams p, SoftmaxParams a) {
  __shared__ CandEntry tab[128];
  __shared__ float thr[128];
  const float g = __fdiv_rn(1.0f, kTensorDiv);   // the tensor scale of numerators whose maximum is 1
  build_cand_entries(tab, g);
  build_c0_thresholds(thr, g);
  __syncthreads();
  const float inv6g = __frcp_rn(__fmul_rn(6.0f, g));
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.gscale_out = g;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t bpr = a.Tk / 16;
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
    for (int64_t j = lane; j < bpr; j += 32) {
      float x[16];
      load_block<DT_F32>(reinterpret_cast<const char*>(sr + 16 * j), a.v8 != 0, x);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        x[i] = 16 * j + i <= lim ? exp_ss(__fsub_rn(x[i], m)) : 0.0f;
        l = __fadd_rn(l, x[i]);
      }
      u64 x2[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) x2[k] = pk2(x[2 * k], x[2 * k + 1]);
      const int64_t b = row * bpr + j;
      if (quantize_block_fast<SRC_LINEAR, false, NC, false>(p, tab, thr, inv6g, false, b, x2))
        quantize_block_def_x2<SRC_LINEAR, false>(p, tab, thr, inv6g, false, b, x2);
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
