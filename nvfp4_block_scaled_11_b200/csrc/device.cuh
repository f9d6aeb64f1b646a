// device.cuh -- sm_100a device helpers for libnvfp4: vector loads/stores, the hardware E2M1 / E4M3
// converters, element widening, and the FWHT-16 butterfly.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

enum : int { DT_F32 = 0, DT_BF16 = 1, DT_F16 = 2 };

// ---- packed FP32x2 arithmetic: each lane rounds exactly as the scalar operation ----
typedef unsigned long long u64;

__device__ __forceinline__ u64 pk2(float lo, float hi) {
  u64 r;
  asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(u64 v, float& lo, float& hi) {
  asm("mov.b64 {%0,%1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ u64 mul2(u64 a, u64 b) {
  u64 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 add2(u64 a, u64 b) {
  u64 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 sub2(u64 a, u64 b) {
  u64 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
  u64 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// ---- streaming loads: read-only path, no L1 allocation (every byte is read once per pass) ----
__device__ __forceinline__ void ld_v8(const void* p, uint32_t (&v)[8]) {
  asm("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
      : "l"(p));
}
__device__ __forceinline__ void ld_v4(const void* p, uint32_t* v) {
  asm("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
      : "l"(p));
}
__device__ __forceinline__ void st_v8(void* p, const uint32_t (&v)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void st_v8(void* p, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void st_v4(void* p, const uint32_t* v) {
  asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
               : "memory");
}

// ---- E2M1 (FP4) converters ----
// Round-to-nearest-even, saturating at +-6, sign kept: returns (E2M1(hi) << 4) | E2M1(lo).
__device__ __forceinline__ uint32_t e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u32.u8 %0, t; }" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Byte of two E2M1 codes -> f16x2 holding their exact values (low nibble -> low half).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t q) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(r) : "r"(q));
  return r;
}
__device__ __forceinline__ float f16lo(uint32_t h2) { return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))); }
__device__ __forceinline__ float f16hi(uint32_t h2) { return __half2float(__ushort_as_half((unsigned short)(h2 >> 16))); }

// ---- E4M3 (FP8) converters ----
// Code of a non-negative, non-NaN value: RNE, saturating at 448 (values >= 448, +Inf -> 0x7E).
__device__ __forceinline__ int e4m3_code(float v) {
  v = fminf(v, 448.0f);
  uint32_t r;
  asm("{ .reg .b16 t; cvt.rn.satfinite.e4m3x2.f32 t, %1, %1; cvt.u32.u16 %0, t; }" : "=r"(r) : "f"(v));
  return (int)(r & 0xFFu);
}
// Exact value of an E4M3 code (0x7F / 0xFF -> NaN).  The code is duplicated into both bytes so the
// result does not depend on which byte feeds which half.
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t b = (code & 0xFFu) * 0x0101u, h2;
  asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h2) : "r"(b));
  return f16lo(h2);
}

// ---- element widening (exact) ----
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int DT>
__device__ __forceinline__ void widen_words(const uint32_t* w, float* x, int nwords) {
#pragma unroll
  for (int k = 0; k < nwords; ++k) {
    if (DT == DT_F32) {
      x[k] = __uint_as_float(w[k]);
    } else if (DT == DT_BF16) {
      x[2 * k] = bf16lo(w[k]);
      x[2 * k + 1] = bf16hi(w[k]);
    } else {
      x[2 * k] = f16lo(w[k]);
      x[2 * k + 1] = f16hi(w[k]);
    }
  }
}

// Load one 16-element block starting at byte address p (32-byte aligned when v8 is true, else 16).
template <int DT>
__device__ __forceinline__ void load_block(const char* p, bool v8, float (&x)[16]) {
  if (DT == DT_F32) {
    uint32_t w[16];
    if (v8) {
      uint32_t a[8], b[8];
      ld_v8(p, a);
      ld_v8(p + 32, b);
#pragma unroll
      for (int k = 0; k < 8; ++k) { w[k] = a[k]; w[8 + k] = b[k]; }
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) ld_v4(p + 16 * k, w + 4 * k);
    }
    widen_words<DT_F32>(w, x, 16);
  } else {
    uint32_t w[8];
    if (v8) {
      ld_v8(p, w);
    } else {
      ld_v4(p, w);
      ld_v4(p + 16, w + 4);
    }
    widen_words<DT>(w, x, 8);
  }
}

// 16 elements of one column: element i at p + i * stride_bytes (a warp reads consecutive columns).
template <int DT>
__device__ __forceinline__ void load_column(const char* p, int64_t stride_bytes, float (&x)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const char* q = p + i * stride_bytes;
    if (DT == DT_F32) {
      x[i] = __ldg(reinterpret_cast<const float*>(q));
    } else {
      const uint32_t h = __ldg(reinterpret_cast<const unsigned short*>(q));
      x[i] = DT == DT_BF16 ? __uint_as_float(h << 16) : __half2float(__ushort_as_half((unsigned short)h));
    }
  }
}

// 16-point Walsh-Hadamard butterflies (strides 1, 2, 4, 8), then times 1/4; FP32, no contraction.
__device__ __forceinline__ void fwht16(float (&a)[16]) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & h) == 0) {
        float u = a[i], v = a[i + h];
        a[i] = __fadd_rn(u, v);
        a[i + h] = __fsub_rn(u, v);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = __fmul_rn(a[i], 0.25f);
}

// The same transform on 8 packed pairs (x2[k] = elements 2k, 2k+1), with the same additions in the same
// order: stage 1 pairs the two lanes of one register (scalar), stages 2, 4 and 8 pair registers k and
// k + h/2 lane by lane (one FP32x2 add and one subtract per register pair), then the packed x0.25.
__device__ __forceinline__ void fwht16_x2(u64 (&x2)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float u, v;
    upk2(x2[k], u, v);
    x2[k] = pk2(__fadd_rn(u, v), __fsub_rn(u, v));
  }
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if ((k & h) == 0) {
        const u64 u = x2[k], v = x2[k + h];
        x2[k] = add2(u, v);
        x2[k + h] = sub2(u, v);
      }
    }
  }
  const u64 q = pk2(0.25f, 0.25f);
#pragma unroll
  for (int k = 0; k < 8; ++k) x2[k] = mul2(x2[k], q);
}

// fwht16_x2 on 16 values held as floats (packed and unpacked around it).
__device__ __forceinline__ void fwht16_packed(float (&a)[16]) {
  u64 x2[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) x2[k] = pk2(a[2 * k], a[2 * k + 1]);
  fwht16_x2(x2);
#pragma unroll
  for (int k = 0; k < 8; ++k) upk2(x2[k], a[2 * k], a[2 * k + 1]);
}

}  // namespace nvfp4
