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
// One thread per (batch, query, head) keeps the head's CH channels in registers: the location,
// bounds test and bilinear weights of a sampling point are computed once for all channels, each
// corner is one gather of CH/2 code bytes plus CH/16 scale bytes, the block scale is folded into the
// corner weight and the channel updates are packed FP32x2 FMAs.  The full-precision twin (FP32 / F16
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

// acc[k] += cw * (value pair k) for the CH/2 channel pairs of one corner.
template <int VT, int CH>
__device__ __forceinline__ void msda_corner(const MsdaParams& p, int64_t kh, float cw, u64 (&acc)[CH / 2]) {
  if constexpr (VT == MSDA_NVFP4) {
    const uint8_t* cp = p.codes + kh * (CH / 2);
    uint32_t cw32[CH / 8];
    if constexpr (CH == 16) {
      const uint2 v = *reinterpret_cast<const uint2*>(cp);
      cw32[0] = v.x; cw32[1] = v.y;
    } else {
#pragma unroll
      for (int k = 0; k < CH / 32; ++k) {
        const uint4 v = *reinterpret_cast<const uint4*>(cp + 16 * k);
        cw32[4 * k] = v.x; cw32[4 * k + 1] = v.y; cw32[4 * k + 2] = v.z; cw32[4 * k + 3] = v.w;
      }
    }
    const uint8_t* sp = p.scales + kh * (CH / 16);
#pragma unroll
    for (int blk = 0; blk < CH / 16; ++blk) {
      const float s = __fmul_rn(cw, e4m3_value(sp[blk]));   // corner weight x block scale
      const u64 ss = pk2(s, s);
#pragma unroll
      for (int k = 0; k < 8; ++k) {                            // byte k of the block: channels 2k, 2k+1
        const uint32_t byte = (cw32[2 * blk + (k >> 2)] >> (8 * (k & 3))) & 0xFFu;
        const uint32_t h2 = e2m1x2_to_f16x2(byte);
        acc[8 * blk + k] = fma2(pk2(f16lo(h2), f16hi(h2)), ss, acc[8 * blk + k]);
      }
    }
  } else if constexpr (VT == MSDA_F32) {
    const float4* vp = reinterpret_cast<const float4*>(p.value + kh * CH * 4);
    const u64 cc = pk2(cw, cw);
#pragma unroll
    for (int k = 0; k < CH / 4; ++k) {
      const float4 v = vp[k];
      acc[2 * k] = fma2(pk2(v.x, v.y), cc, acc[2 * k]);
      acc[2 * k + 1] = fma2(pk2(v.z, v.w), cc, acc[2 * k + 1]);
    }
  } else {
    const uint4* vp = reinterpret_cast<const uint4*>(p.value + kh * CH * 2);
    const u64 cc = pk2(cw, cw);
#pragma unroll
    for (int k = 0; k < CH / 8; ++k) {
      const uint4 v = vp[k];
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = VT == MSDA_F16 ? f16lo(wd[j]) : bf16lo(wd[j]);
        const float hi = VT == MSDA_F16 ? f16hi(wd[j]) : bf16hi(wd[j]);
        acc[4 * k + j] = fma2(pk2(lo, hi), cc, acc[4 * k + j]);
      }
    }
  }
}

template <int VT, int CH>
__global__ void __launch_bounds__(128) msda_forward_kernel(MsdaParams p) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const float g = VT == MSDA_NVFP4 ? *p.gsrc : 1.0f;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < p.total; t += stride) {
    const int64_t h = t % p.heads;
    const int64_t b = t / (p.heads * p.nq);
    u64 acc[CH / 2];
#pragma unroll
    for (int k = 0; k < CH / 2; ++k) acc[k] = 0ull;
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
#pragma unroll
        for (int cy = 0; cy < 2; ++cy) {
          const int yy = y0 + cy;
          if (yy < 0 || yy >= H) continue;
          const float wy = __fmul_rn(wt, cy ? fy : gy);
#pragma unroll
          for (int cx = 0; cx < 2; ++cx) {
            const int xx = x0 + cx;
            if (xx < 0 || xx >= W) continue;
            const float cw = __fmul_rn(wy, cx ? fx : gx);
            msda_corner<VT, CH>(p, (key0 + (int64_t)yy * W + xx) * p.heads + h, cw, acc);
          }
        }
      }
    }
    // write the head's channels (scaled by g for NVFP4): CH * 4 bytes, 32-byte aligned
    float* o = p.out + t * CH;
#pragma unroll
    for (int k = 0; k < CH / 8; ++k) {
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
