// msda.cuh -- multi-scale deformable attention forward reading NVFP4 (ScaleSearch-quantized) values.
//
// "自動運転モデル BEVFormer の NVIDIA Blackwell B200 FP8/FP4 CUDAカーネル・チューニング" (qiita.com), sections 5-7:
// the value tensor is the only low-precision operand; sampling locations, attention weights, the
// bilinear interpolation and the accumulation stay FP32, and two FP4 values are decoded per
// instruction.  Here the values are NVFP4 (16-element blocks along the channels, E4M3 block scales,
// FP32 tensor scale g) as the ScaleSearch quantizer writes them:
//   out[b,q,h,c] = g * sum_l sum_p w * sum_corners bilinear_weight * E2M1(code) * E4M3(block scale)
// with corners outside the level's map contributing zero (sampling at loc * size - 0.5).
//
// A thread owns a slice of whole 16-channel blocks of one (batch, query, head) in registers: the
// location, bounds test and bilinear weights of a sampling point are computed once per slice, each
// corner is one gather of the slice's code bytes plus its scale bytes, the block scale is folded into
// the corner weight and the channel updates are packed FP32x2 FMAs.  The full-precision twin (FP32 / F16
// / BF16 values) runs the same loop on plain values, for the footprint / speed comparison.
#pragma once

#include "search.cuh"

namespace nvfp4 {

constexpr int kMsdaMaxLevels = 8;
enum { MSDA_NVFP4 = 0, MSDA_F32 = 1, MSDA_F16 = 2, MSDA_BF16 = 3 };

struct MsdaParams {
  const uint8_t* codes;    // NVFP4: [bs, nkeys, heads, CH/2]
  const uint8_t* scales;   // NVFP4: [bs, nkeys, heads, CH/16] E4M3 block scales
  const float* gsrc;       // NVFP4: tensor scale (device)
  const char* value;       // twin: [bs, nkeys, heads, CH] FP32 / F16 / BF16
  const float* loc;        // [bs, nq, heads, L, P, 2]
  const float* w;          // [bs, nq, heads, L, P]
  float* out;              // [bs, nq, heads, CH]
  int64_t nkeys, heads, nq, total;  // total = bs * nq * heads
  int L, P;
  int H[kMsdaMaxLevels], W[kMsdaMaxLevels];
  int64_t start[kMsdaMaxLevels];
};

// Raw bytes of one corner's channel slice [coff, coff + CHT) (kh = key * heads + head): loaded for all
// four corners of a sampling point before any of them is used, so the gathers overlap.
template <int VT, int CHT>
struct CornerData {
  static constexpr int kWords = VT == MSDA_NVFP4 ? CHT / 8 : (VT == MSDA_F32 ? CHT : CHT / 2);
  uint32_t w[kWords];
  uint32_t sc;  // NVFP4: the CHT/16 scale bytes (little-endian)
};

template <int VT, int CH, int CHT>
__device__ __forceinline__ void msda_load(const MsdaParams& p, int64_t kh, int coff, CornerData<VT, CHT>& d) {
  if constexpr (VT == MSDA_NVFP4) {
    const uint8_t* cp = p.codes + kh * (CH / 2) + coff / 2;
    if constexpr (CHT == 16) {
      const uint2 v = *reinterpret_cast<const uint2*>(cp);
      d.w[0] = v.x; d.w[1] = v.y;
    } else {
#pragma unroll
      for (int k = 0; k < CHT / 32; ++k) {
        const uint4 v = *reinterpret_cast<const uint4*>(cp + 16 * k);
        d.w[4 * k] = v.x; d.w[4 * k + 1] = v.y; d.w[4 * k + 2] = v.z; d.w[4 * k + 3] = v.w;
      }
    }
    const uint8_t* sp = p.scales + kh * (CH / 16) + coff / 16;
    d.sc = 0u;
#pragma unroll
    for (int blk = 0; blk < CHT / 16; ++blk) d.sc |= (uint32_t)sp[blk] << (8 * blk);
  } else {
    constexpr int ES = VT == MSDA_F32 ? 4 : 2;
    const uint4* vp = reinterpret_cast<const uint4*>(p.value + (kh * CH + coff) * ES);
#pragma unroll
    for (int k = 0; k < CornerData<VT, CHT>::kWords / 4; ++k) {
      const uint4 v = vp[k];
      d.w[4 * k] = v.x; d.w[4 * k + 1] = v.y; d.w[4 * k + 2] = v.z; d.w[4 * k + 3] = v.w;
    }
  }
}

// acc[k] += cw * (value pair k) for the CHT/2 channel pairs of one loaded corner.
template <int VT, int CHT>
__device__ __forceinline__ void msda_accumulate(const CornerData<VT, CHT>& d, float cw, u64 (&acc)[CHT / 2]) {
  if constexpr (VT == MSDA_NVFP4) {
#pragma unroll
    for (int blk = 0; blk < CHT / 16; ++blk) {
      const float s = __fmul_rn(cw, e4m3_value((d.sc >> (8 * blk)) & 0xFFu));   // corner weight x block scale
      const u64 ss = pk2(s, s);
#pragma unroll
      for (int k = 0; k < 8; ++k) {                                             // channels 2k, 2k+1 of the block
        const uint32_t byte = (d.w[2 * blk + (k >> 2)] >> (8 * (k & 3))) & 0xFFu;
        const uint32_t h2 = e2m1x2_to_f16x2(byte);
        acc[8 * blk + k] = fma2(pk2(f16lo(h2), f16hi(h2)), ss, acc[8 * blk + k]);
      }
    }
  } else {
    const u64 cc = pk2(cw, cw);
#pragma unroll
    for (int k = 0; k < CHT / 2; ++k) {
      float lo, hi;
      if (VT == MSDA_F32) {
        lo = __uint_as_float(d.w[2 * k]);
        hi = __uint_as_float(d.w[2 * k + 1]);
      } else if (VT == MSDA_F16) {
        lo = f16lo(d.w[k]);
        hi = f16hi(d.w[k]);
      } else {
        lo = bf16lo(d.w[k]);
        hi = bf16hi(d.w[k]);
      }
      acc[k] = fma2(pk2(lo, hi), cc, acc[k]);
    }
  }
}

// SPLIT threads share one (batch, query, head), each owning CH / SPLIT consecutive channels (whole
// 16-channel blocks).
template <int VT, int CH, int SPLIT>
__global__ void __launch_bounds__(128) msda_forward_kernel(MsdaParams p) {
  constexpr int CHT = CH / SPLIT;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const float g = VT == MSDA_NVFP4 ? *p.gsrc : 1.0f;
  const int64_t nthreads = p.total * SPLIT;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < nthreads; u += stride) {
    const int64_t t = u / SPLIT;
    const int coff = (int)(u - t * SPLIT) * CHT;
    const int64_t h = t % p.heads;
    const int64_t b = t / (p.heads * p.nq);
    u64 acc[CHT / 2];
#pragma unroll
    for (int k = 0; k < CHT / 2; ++k) acc[k] = 0ull;
    const float* lp = p.loc + t * p.L * p.P * 2;
    const float* wp = p.w + t * p.L * p.P;
    for (int l = 0; l < p.L; ++l) {
      const int H = p.H[l], W = p.W[l];
      const int64_t key0 = b * p.nkeys + p.start[l];
      for (int pt = 0; pt < p.P; ++pt) {
        const int i = l * p.P + pt;
        const float x = __fsub_rn(__fmul_rn(lp[2 * i], (float)W), 0.5f);
        const float y = __fsub_rn(__fmul_rn(lp[2 * i + 1], (float)H), 0.5f);
        if (!(x > -1.0f && y > -1.0f && x < (float)W && y < (float)H)) continue;
        const float wt = wp[i];
        const float xf = floorf(x), yf = floorf(y);
        const int x0 = (int)xf, y0 = (int)yf;
        const float fx = __fsub_rn(x, xf), fy = __fsub_rn(y, yf);
        const float gx = __fsub_rn(1.0f, fx), gy = __fsub_rn(1.0f, fy);
        // the four corners: off-map ones read an on-map address and are skipped when accumulating
        CornerData<VT, CHT> d[4];
        bool ok[4];
        float cw[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int yy = y0 + (c >> 1), xx = x0 + (c & 1);
          ok[c] = yy >= 0 && yy < H && xx >= 0 && xx < W;
          const int ys = min(max(yy, 0), H - 1), xs = min(max(xx, 0), W - 1);
          cw[c] = __fmul_rn(__fmul_rn(wt, (c >> 1) ? fy : gy), (c & 1) ? fx : gx);
          msda_load<VT, CH, CHT>(p, (key0 + (int64_t)ys * W + xs) * p.heads + h, coff, d[c]);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (ok[c]) msda_accumulate<VT, CHT>(d[c], cw[c], acc);
      }
    }
    // write this thread's channels (scaled by g for NVFP4): CHT * 4 bytes, 32-byte aligned
    float* o = p.out + t * CH + coff;
#pragma unroll
    for (int k = 0; k < CHT / 8; ++k) {
      uint32_t v[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float lo, hi;
        upk2(acc[4 * k + j], lo, hi);
        v[2 * j] = __float_as_uint(__fmul_rn(lo, g));
        v[2 * j + 1] = __float_as_uint(__fmul_rn(hi, g));
      }
      st_v8(o + 8 * k, v);
    }
  }
}

}  // namespace nvfp4
