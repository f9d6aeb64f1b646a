// kernels.cuh -- libnvfp4 kernels for sm_100a: tensor amax, ScaleSearch quantize, dequantize,
// Hadamard-16 and the pieces of the mixed-precision KV layout.
//
// Sources (web pages, by title and section):
//   "NVIDIAのFP4推論が50倍の効率を実現" (introl.com), 超低精度推論を支えるアーキテクチャ: the NVFP4 format.
//   "Search your block floating-point scales!" (gist.science summary of arXiv 2605.12464),
//     Method > ScaleSearch: the scale search; ScaleSearchAttention: Hadamard rotation, sink/recent KV.
//   "BEVFormer on B200: FP8/FP4 CUDA kernel tuning" (qiita.com), section 7: scale applied back by one
//     multiply; two FP4 codes per byte.
#pragma once

#include <float.h>

#include "device.cuh"

namespace nvfp4 {

constexpr float kTensorDiv = 2688.0f;  // 6 (largest E2M1) * 448 (largest E4M3)

// =================================================================================================
// Tensor amax: unsigned max of the magnitude bits (NaN > Inf > finite, so both propagate), reduced
// per CTA and merged with one atomicMax into a caller word that was zeroed beforehand.
// =================================================================================================
template <int DT>
__device__ __forceinline__ uint32_t mag_max_words(const uint32_t* w, int nw, uint32_t m) {
#pragma unroll
  for (int k = 0; k < nw; ++k) {
    if (DT == DT_F32) m = max(m, w[k] & 0x7FFFFFFFu);
    else m = __vmaxu2(m, w[k] & 0x7FFF7FFFu);  // two 16-bit magnitudes per word
  }
  return m;
}

template <int DT>
__device__ __forceinline__ uint32_t mag_to_f32bits(uint32_t m) {
  if (DT == DT_F32) return m;
  uint32_t h = max(m & 0xFFFFu, m >> 16);
  if (DT == DT_BF16) return h << 16;
  return __float_as_uint(__half2float(__ushort_as_half((unsigned short)h)));
}

template <int DT>
__global__ void __launch_bounds__(512) amax_kernel(const char* __restrict__ x, int64_t n, int v8,
                                                   uint32_t* __restrict__ out) {
  constexpr int ES = DT == DT_F32 ? 4 : 2;
  constexpr int EPV = 32 / ES;  // elements per 32-byte vector
  const int64_t nvec = n / EPV;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t m = 0;
  if (v8) {
    for (; i + 3 * stride < nvec; i += 4 * stride) {
      uint32_t a[8], b[8], c[8], d[8];
      ld_v8(x + 32 * i, a);
      ld_v8(x + 32 * (i + stride), b);
      ld_v8(x + 32 * (i + 2 * stride), c);
      ld_v8(x + 32 * (i + 3 * stride), d);
      m = mag_max_words<DT>(a, 8, m);
      m = mag_max_words<DT>(b, 8, m);
      m = mag_max_words<DT>(c, 8, m);
      m = mag_max_words<DT>(d, 8, m);
    }
    for (; i < nvec; i += stride) {
      uint32_t a[8];
      ld_v8(x + 32 * i, a);
      m = mag_max_words<DT>(a, 8, m);
    }
  } else {
    for (; i < nvec; i += stride) {
      uint32_t a[4], b[4];
      ld_v4(x + 32 * i, a);
      ld_v4(x + 32 * i + 16, b);
      m = mag_max_words<DT>(a, 4, m);
      m = mag_max_words<DT>(b, 4, m);
    }
  }
  m = mag_to_f32bits<DT>(m);
  // ragged tail (n % EPV elements), one element per thread of the first CTA
  if (blockIdx.x == 0) {
    const int64_t t = nvec * EPV + threadIdx.x;
    if (t < n) {
      uint32_t b;
      if (DT == DT_F32) b = reinterpret_cast<const uint32_t*>(x)[t] & 0x7FFFFFFFu;
      else {
        uint32_t h = reinterpret_cast<const uint16_t*>(x)[t] & 0x7FFFu;
        b = mag_to_f32bits<DT>(h);
      }
      m = max(m, b);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t s[32];
  if ((threadIdx.x & 31) == 0) s[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? s[threadIdx.x] : 0u;
#pragma unroll
    for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (threadIdx.x == 0 && m) atomicMax(out, m);
  }
}

// g = fl(amax / 2688), in place or into another word.
__global__ void global_scale_kernel(const float* amax, float* g) {
  if (threadIdx.x == 0 && blockIdx.x == 0) *g = __fdiv_rn(*amax, kTensorDiv);
}

// =================================================================================================
// ScaleSearch quantize.
// =================================================================================================
struct QuantParams {
  const char* x;       // input base (bytes)
  int64_t nblocks;
  int f_lo, f_hi;
  const float* g_src;  // device word: g itself, or the tensor amax when g_is_amax
  int g_is_amax;
  uint8_t* codes;
  uint8_t* scales;
  int8_t* block_f;     // optional
  float* block_sse;    // optional
  int v8;              // input base is 32-byte aligned
  // mixed KV layout: blocks run over the middle tokens of K[BH, T, D]
  int64_t T, Tm, sink, D, bpr;  // bpr = D / 16
  // scales in the tensor-core tile layout when sf_bpr > 0: the blocks form matrices of sf_rows rows and
  // sf_bpr blocks per row (fewer than 2^32 blocks in all); each matrix's scales take sf_mat_bytes bytes
  uint32_t sf_bpr, sf_rows, sf_ctiles;  // sf_ctiles = ceil(sf_bpr / 4)
  int64_t sf_mat_bytes;
  // KV append: when out_cap > 0 the Tm token rows of each (batch, head) handled by this launch are
  // written to rows out_t0 .. out_t0 + Tm - 1 of a cache with out_cap rows per (batch, head)
  int64_t out_cap, out_t0;
  // column blocks (source mode SRC_COLS): x is [batch, rows, tr_cols] and a block is 16 consecutive
  // rows of one column; tr_rb = rows / 16.  Blocks run column-fastest, so a warp reads rows of
  // consecutive columns; outputs are the transposed [batch, tr_cols, rows] layout.
  int64_t tr_cols, tr_rb;
  // fused round trip (linear mode): when deq_out is set, each block's dequantized values (the input's
  // dtype) are written there too, at the block's own position
  char* deq_out;
  int deq_v8;          // deq_out is 32-byte aligned
};

// Where the 16 elements of a block come from.
enum { SRC_LINEAR = 0, SRC_KV = 1, SRC_COLS = 2 };

// Column-mode block b -> (batch l, column c, row block rb); fewer than 2^32 blocks (host-checked).
__device__ __forceinline__ void cols_split(const QuantParams& p, int64_t b, uint32_t& l, uint32_t& c, uint32_t& rb) {
  const uint32_t ub = (uint32_t)b, C = (uint32_t)p.tr_cols, RB = (uint32_t)p.tr_rb;
  const uint32_t rest = ub / C;
  c = ub - rest * C;
  l = rest / RB;
  rb = rest - l * RB;
}

// KV launches cover fewer than 2^32 blocks (checked by the host), so block indices split with 32-bit
// arithmetic: block b is (bh, t, j) = (head row, middle token, block column).
__device__ __forceinline__ void kv_split(int64_t b, int64_t Tm, int64_t bpr, uint32_t& bh, uint32_t& t, uint32_t& j) {
  const uint32_t ub = (uint32_t)b, per = (uint32_t)(Tm * bpr), ubpr = (uint32_t)bpr;
  bh = ub / per;
  const uint32_t rem = ub - bh * per;
  t = rem / ubpr;
  j = rem - t * ubpr;
}

// Element offset of KV block b in K[BH, T, D]: middle token t of head row bh, block column j.
__device__ __forceinline__ int64_t kv_block_elem(int64_t b, int64_t Tm, int64_t bpr, int64_t T, int64_t sink,
                                                 int64_t D) {
  uint32_t bh, t, j;
  kv_split(b, Tm, bpr, bh, t, j);
  return ((int64_t)bh * T + sink + t) * D + 16 * (int64_t)j;
}

// The split (bh, t, j) of KV block indices along a grid-stride loop: one division-based split at the
// first block, then each step adds the stride, written as (qt head rows, qr tokens, rs block columns),
// with at most one carry per level, so the loop itself divides nothing.
struct KvCursor {
  uint32_t bh, t, j;
  uint32_t qt, qr, rs, Tm, bpr;
  __device__ __forceinline__ void init(int64_t b, int64_t stride, int64_t Tm_, int64_t bpr_) {
    Tm = (uint32_t)Tm_;
    bpr = (uint32_t)bpr_;
    kv_split(b, Tm_, bpr_, bh, t, j);
    const uint32_t S = (uint32_t)stride, qs = S / bpr;
    rs = S - qs * bpr;
    qt = qs / Tm;
    qr = qs - qt * Tm;
  }
  __device__ __forceinline__ void advance() {
    j += rs;
    const uint32_t c = j >= bpr ? 1u : 0u;
    j -= c * bpr;
    uint64_t tt = (uint64_t)t + qr + c;   // < 2 Tm
    bh += qt;
    if (tt >= Tm) {
      tt -= Tm;
      ++bh;
    }
    t = (uint32_t)tt;
  }
  __device__ __forceinline__ int64_t elem(int64_t T, int64_t sink, int64_t D) const {
    return ((int64_t)bh * T + sink + t) * D + 16 * (int64_t)j;
  }
};

// Output block index of block b (input order), fixed by the source mode at compile time: linear blocks
// land where they are read; KV blocks land in rows out_t0.. of a cap-row cache when appending
// (out_cap > 0); column blocks land in the transposed layout (row c of matrix l, block rb).
template <int MODE>
__device__ __forceinline__ int64_t out_block(const QuantParams& p, int64_t b) {
  if constexpr (MODE == SRC_COLS) {
    uint32_t l, c, rb;
    cols_split(p, b, l, c, rb);
    return ((int64_t)l * p.tr_cols + c) * p.tr_rb + rb;
  } else if constexpr (MODE == SRC_KV) {
    if (p.out_cap == 0) return b;
    uint32_t bh, t, j;
    kv_split(b, p.Tm, p.bpr, bh, t, j);
    return ((int64_t)bh * p.out_cap + p.out_t0 + t) * p.bpr + j;
  } else {
    return b;
  }
}

// Byte of block b's scale.  Linear: b.  Tile layout (block-scaled tensor-core MMA operand): 512-byte
// tiles of 128 rows x 4 block columns, the column tiles of a row tile consecutive, and inside a tile
// row r, column c at 16 * (r mod 32) + 4 * (r div 32) + c.
__device__ __forceinline__ int64_t scale_index(const QuantParams& p, int64_t b) {
  if (p.sf_bpr == 0u) return b;
  const uint32_t ub = (uint32_t)b, per = p.sf_rows * p.sf_bpr;
  const uint32_t mat = ub / per, rem = ub - mat * per;
  const uint32_t r = rem / p.sf_bpr, c = rem - r * p.sf_bpr;
  const uint32_t in_mat = ((r >> 7) * p.sf_ctiles + (c >> 2)) * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + (c & 3u);
  return (int64_t)mat * p.sf_mat_bytes + in_mat;
}

// Candidate table for one launch: d[c] = fl(E4M3(c) * g), r[c] = fl(1 / d[c]); r = 0 marks a code that
// cannot be a scale (c outside 1..126, d == 0 or 1/d not finite).
struct CandTable {
  float d[128];
  float r[128];
};

__device__ __forceinline__ void build_cand_table(CandTable& t, float g) {
  for (int c = threadIdx.x; c < 128; c += blockDim.x) {
    float d = __fmul_rn(e4m3_value((uint32_t)c), g);
    float r = __frcp_rn(d);
    bool ok = c >= 1 && c <= 126 && d != 0.0f && fabsf(r) <= FLT_MAX;
    t.d[c] = d;
    t.r[c] = ok ? r : 0.0f;
  }
}

// Block squared error of candidate (d, r), summed in FP32 in element order (the definition).
__device__ __forceinline__ float block_sse_exact(const float (&a)[16], float d, float r) {
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    float y0 = __fmul_rn(a[i], r), y1 = __fmul_rn(a[i + 1], r);
    uint32_t h2 = e2m1x2_to_f16x2(e2m1x2(y1, y0));
    float e0 = __fsub_rn(a[i], __fmul_rn(f16lo(h2), d));
    float e1 = __fsub_rn(a[i + 1], __fmul_rn(f16hi(h2), d));
    s = __fadd_rn(s, __fmul_rn(e0, e0));
    s = __fadd_rn(s, __fmul_rn(e1, e1));
  }
  return s;
}

template <int DT, int MODE, bool ROT>
__global__ void __launch_bounds__(256) quantize_kernel(QuantParams p) {
  __shared__ CandTable tab;
  float g = *p.g_src;
  if (p.g_is_amax) g = __fdiv_rn(g, kTensorDiv);
  const bool g_bad = !(g >= 0.0f) || !(g <= FLT_MAX);  // NaN, Inf or negative
  build_cand_table(tab, g);
  __syncthreads();

  constexpr int ES = DT == DT_F32 ? 4 : 2;
  const int span = max(abs(p.f_lo), abs(p.f_hi));
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < p.nblocks; b += stride) {
    float x[16];
    if (MODE == SRC_COLS) {
      uint32_t l, c, rb;
      cols_split(p, b, l, c, rb);
      load_column<DT>(p.x + (((int64_t)l * p.tr_rb + rb) * 16 * p.tr_cols + c) * ES, p.tr_cols * ES, x);
    } else {
      const int64_t elem = MODE == SRC_KV ? kv_block_elem(b, p.Tm, p.bpr, p.T, p.sink, p.D) : 16 * b;
      load_block<DT>(p.x + elem * ES, p.v8 != 0, x);
    }
    if (ROT) fwht16(x);

    float a[16];
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      a[i] = fabsf(x[i]);
      m = max(m, __float_as_uint(x[i]) & 0x7FFFFFFFu);
    }

    uint32_t lo = 0, hi = 0;  // packed codes
    int scale, fstar = -128;
    float sse;
    if (g_bad || m >= 0x7F800000u) {  // poisoned block
      scale = 0x7F;
      sse = __uint_as_float(0x7FFFFFFFu);
    } else {
      float best = 0.0f;
      int c0 = 0;
      if (m != 0) {
        const float t = __fdiv_rn(__uint_as_float(m), 6.0f);
        c0 = e4m3_code(__fdiv_rn(t, g));
        for (int jv = 0; jv <= 2 * span; ++jv) {
          const int f = (jv == 0) ? 0 : ((jv & 1) ? -((jv + 1) >> 1) : (jv >> 1));
          if (f < p.f_lo || f > p.f_hi) continue;
          const int c = c0 + f;
          if (c < 1 || c > 126) continue;
          const float r = tab.r[c];
          if (r == 0.0f) continue;
          const float s = block_sse_exact(a, tab.d[c], r);
          if (fstar == -128 || s < best) {
            best = s;
            fstar = f;
          }
        }
      }
      if (fstar != -128) {
        const int cs = c0 + fstar;
        const float r = tab.r[cs];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          lo |= (e2m1x2(__fmul_rn(x[2 * k + 1], r), __fmul_rn(x[2 * k], r)) & 0xFFu) << (8 * k);
          hi |= (e2m1x2(__fmul_rn(x[2 * k + 9], r), __fmul_rn(x[2 * k + 8], r)) & 0xFFu) << (8 * k);
        }
        scale = cs;
        sse = best;
      } else {
        // zero block, or no usable candidate: sign-only zero codes, scale 0
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          uint32_t nib = ((__float_as_uint(x[2 * k]) >> 31) << 3) | ((__float_as_uint(x[2 * k + 1]) >> 31) << 7);
          if (k < 4) lo |= nib << (8 * k);
          else hi |= nib << (8 * (k - 4));
        }
        scale = 0;
        float s = 0.0f;
        if (m != 0) {
#pragma unroll
          for (int i = 0; i < 16; ++i) s = __fadd_rn(s, __fmul_rn(x[i], x[i]));
        }
        sse = s;
      }
    }
    const int64_t ob = out_block<MODE>(p, b);
    reinterpret_cast<uint2*>(p.codes)[ob] = make_uint2(lo, hi);
    p.scales[scale_index(p, ob)] = (uint8_t)scale;
    if (p.block_f) p.block_f[ob] = (int8_t)fstar;
    if (p.block_sse) p.block_sse[ob] = sse;
  }
}

// =================================================================================================
// Dequantize: one thread per block; the block step d = fl(E4M3(scale) * g) is applied by one multiply.
// =================================================================================================
// The 16 values of one block from its packed codes (cw_lo: elements 0..7, cw_hi: 8..15) and its step
// d = fl(E4M3(scale) * g): out_i = fl(E2M1(q_i) * d), narrowed to OT by RNE, stored at o (64 bytes for
// FP32, 32 otherwise; v8: o is 32-byte aligned).  Shared by the dequantize kernel and the fused round
// trip, so the two agree bit for bit.
template <int OT>
__device__ __forceinline__ void store_dequantized(char* o, uint32_t cw_lo, uint32_t cw_hi, float d, bool v8) {
  float v[16];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t byte = ((k < 4 ? cw_lo : cw_hi) >> (8 * (k & 3))) & 0xFFu;
    const uint32_t h2 = e2m1x2_to_f16x2(byte);
    v[2 * k] = __fmul_rn(f16lo(h2), d);
    v[2 * k + 1] = __fmul_rn(f16hi(h2), d);
  }
  if (OT == DT_F32) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(v[i]);
    if (v8) {
      st_v8(o, static_cast<const uint32_t*>(w));
      st_v8(o + 32, w + 8);
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) st_v4(o + 16 * k, w + 4 * k);
    }
  } else {
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (OT == DT_BF16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
        w[k] = *reinterpret_cast<uint32_t*>(&h);
      } else {
        __half2 h = __floats2half2_rn(v[2 * k], v[2 * k + 1]);
        w[k] = *reinterpret_cast<uint32_t*>(&h);
      }
    }
    if (v8) {
      st_v8(o, w);
    } else {
      st_v4(o, w);
      st_v4(o + 16, w + 4);
    }
  }
}

template <int OT>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t* __restrict__ codes,
                                                         const uint8_t* __restrict__ scales,
                                                         const float* __restrict__ gsrc, int64_t nblocks,
                                                         char* __restrict__ out, int v8) {
  constexpr int OS = OT == DT_F32 ? 4 : 2;
  const float g = *gsrc;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
    const uint2 cw = reinterpret_cast<const uint2*>(codes)[b];
    store_dequantized<OT>(out + 16 * OS * b, cw.x, cw.y, __fmul_rn(e4m3_value(scales[b]), g), v8 != 0);
  }
}

// =================================================================================================
// Hadamard-16: one thread per group of 16.  An optional sign diagonal D (bit i of `signs` negates
// element i, exactly, by flipping its sign bit) goes before the butterflies (H D) or, for the inverse,
// after them (D H).
// =================================================================================================
__device__ __forceinline__ void flip_signs(float (&a)[16], const uint32_t (&m)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = __uint_as_float(__float_as_uint(a[i]) ^ m[i]);
}

template <int DT, int OT>
__global__ void __launch_bounds__(256) hadamard16_kernel(const char* __restrict__ x, int64_t ngroups,
                                                         char* __restrict__ out, int v8_in, int v8_out,
                                                         uint32_t signs, int inverse) {
  constexpr int ES = DT == DT_F32 ? 4 : 2;
  constexpr int OS = OT == DT_F32 ? 4 : 2;
  uint32_t m[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) m[i] = ((signs >> i) & 1u) << 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < ngroups; b += stride) {
    float a[16];
    load_block<DT>(x + 16 * ES * b, v8_in != 0, a);
    if (!inverse) flip_signs(a, m);
    fwht16_packed(a);
    if (inverse) flip_signs(a, m);
    char* o = out + 16 * OS * b;
    if (OT == DT_F32) {
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(a[i]);
      if (v8_out) {
        st_v8(o, static_cast<const uint32_t*>(w));
        st_v8(o + 32, w + 8);
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) st_v4(o + 16 * k, w + 4 * k);
      }
    } else {
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (OT == DT_BF16) {
          __nv_bfloat162 h = __floats2bfloat162_rn(a[2 * k], a[2 * k + 1]);
          w[k] = *reinterpret_cast<uint32_t*>(&h);
        } else {
          __half2 h = __floats2half2_rn(a[2 * k], a[2 * k + 1]);
          w[k] = *reinterpret_cast<uint32_t*>(&h);
        }
      }
      if (v8_out) {
        st_v8(o, w);
      } else {
        st_v4(o, w);
        st_v4(o + 16, w + 4);
      }
    }
  }
}

// =================================================================================================
// MXFP4 (the power-of-two-scaled format NVFP4 is compared against): OCP Microscaling v1.0 -- blocks of
// 32, one E8M0 scale 2^e with e = floor(log2 amax_b) - 2 (clamped to [-127, 127]), elements
// E2M1_RNE_SAT(x * 2^-e); all-zero block e = -127; a NaN / Inf element -> scale 0xFF, codes 0.
// =================================================================================================
// 2^k as an exact float for k in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float pow2_exact(int k) {
  return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(1u << (k + 149));
}

template <int DT>
__global__ void __launch_bounds__(256) mxfp4_quantize_kernel(const char* __restrict__ x, int64_t nblocks, int v8,
                                                             uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  constexpr int ES = DT == DT_F32 ? 4 : 2;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
    float v0[16], v1[16];
    load_block<DT>(x + 32 * ES * b, v8 != 0, v0);
    load_block<DT>(x + 32 * ES * b + 16 * ES, v8 != 0, v1);
    uint32_t mb = 0u;  // largest magnitude bit pattern: integer order = numeric order; NaN / Inf >= 0x7F800000
#pragma unroll
    for (int i = 0; i < 16; ++i) mb = max(mb, max(__float_as_uint(v0[i]) & 0x7FFFFFFFu, __float_as_uint(v1[i]) & 0x7FFFFFFFu));
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    int sbyte = 0xFF;
    if (mb < 0x7F800000u) {
      const int ex = (int)(mb >> 23);
      int e = mb == 0u ? -127 : (ex > 0 ? ex - 127 : (31 - __clz((int)mb)) - 149) - 2;
      e = max(e, -127);
      sbyte = e + 127;
      const float inv = pow2_exact(-e);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float lo = k < 8 ? v0[2 * k] : v1[2 * k - 16], hi = k < 8 ? v0[2 * k + 1] : v1[2 * k - 15];
        w[k >> 2] |= (e2m1x2(__fmul_rn(hi, inv), __fmul_rn(lo, inv)) & 0xFFu) << (8 * (k & 3));
      }
    }
    reinterpret_cast<uint4*>(codes)[b] = make_uint4(w[0], w[1], w[2], w[3]);
    scales[b] = (uint8_t)sbyte;
  }
}

template <int OT>
__device__ __forceinline__ void store16(char* o, const float (&v)[16], bool v8) {
  if (OT == DT_F32) {
    uint32_t a[8], c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { a[i] = __float_as_uint(v[i]); c[i] = __float_as_uint(v[8 + i]); }
    if (v8) {
      st_v8(o, a);
      st_v8(o + 32, c);
    } else {
      st_v4(o, a); st_v4(o + 16, a + 4); st_v4(o + 32, c); st_v4(o + 48, c + 4);
    }
  } else {
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (OT == DT_BF16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
        w[k] = *reinterpret_cast<uint32_t*>(&h);
      } else {
        __half2 h = __floats2half2_rn(v[2 * k], v[2 * k + 1]);
        w[k] = *reinterpret_cast<uint32_t*>(&h);
      }
    }
    if (v8) {
      st_v8(o, w);
    } else {
      st_v4(o, w);
      st_v4(o + 16, w + 4);
    }
  }
}

template <int OT>
__global__ void __launch_bounds__(256) mxfp4_dequantize_kernel(const uint8_t* __restrict__ codes,
                                                               const uint8_t* __restrict__ scales, int64_t nblocks,
                                                               char* __restrict__ out, int v8) {
  constexpr int OS = OT == DT_F32 ? 4 : 2;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
    const uint4 cw = reinterpret_cast<const uint4*>(codes)[b];
    const uint32_t s = scales[b];
    const float X = s == 0xFFu ? __uint_as_float(0x7FC00000u) : pow2_exact((int)s - 127);
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float v[16];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t byte = (words[2 * half + (k >> 2)] >> (8 * (k & 3))) & 0xFFu;
        const uint32_t h2 = e2m1x2_to_f16x2(byte);
        v[2 * k] = __fmul_rn(f16lo(h2), X);
        v[2 * k + 1] = __fmul_rn(f16hi(h2), X);
      }
      store16<OT>(out + (32 * b + 16 * half) * OS, v, v8 != 0);
    }
  }
}

// =================================================================================================
// Mixed-precision KV layout helpers.
// =================================================================================================
// Copy the first `sink` and last `recent` token rows of every (batch, head) verbatim (16-byte units).
__global__ void __launch_bounds__(256) kv_copy_kernel(const char* __restrict__ k, int64_t BH, int64_t T,
                                                      int64_t row_bytes, int64_t sink, int64_t recent,
                                                      char* __restrict__ sink_out, char* __restrict__ recent_out) {
  const int64_t units_per_row = row_bytes / 16;
  const int64_t per_bh = (sink + recent) * units_per_row;
  const int64_t total = BH * per_bh;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += stride) {
    const int64_t bh = u / per_bh;
    const int64_t r = u - bh * per_bh;
    const int64_t tok = r / units_per_row;
    const int64_t w = r - tok * units_per_row;
    const char* src;
    char* dst;
    if (tok < sink) {
      src = k + ((bh * T + tok) * row_bytes) + 16 * w;
      dst = sink_out + ((bh * sink + tok) * row_bytes) + 16 * w;
    } else {
      const int64_t tr = tok - sink;
      src = k + ((bh * T + (T - recent) + tr) * row_bytes) + 16 * w;
      dst = recent_out + ((bh * recent + tr) * row_bytes) + 16 * w;
    }
    uint32_t v[4];
    ld_v4(src, v);
    st_v4(dst, v);
  }
}

// amax over the (optionally rotated) middle tokens; one thread per 16-group.
template <bool ROT>
__global__ void __launch_bounds__(256) kv_amax_kernel(const char* __restrict__ k, int64_t ngroups, int64_t T,
                                                      int64_t Tm, int64_t sink, int64_t D, int64_t bpr, int v8,
                                                      uint32_t* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  uint32_t m = 0;
  int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  KvCursor kc;
  if (b < ngroups) kc.init(b, stride, Tm, bpr);
  for (; b < ngroups; b += stride, kc.advance()) {
    float x[16];
    load_block<DT_BF16>(k + 2 * kc.elem(T, sink, D), v8 != 0, x);
    if (ROT) fwht16_packed(x);
#pragma unroll
    for (int i = 0; i < 16; ++i) m = max(m, __float_as_uint(x[i]) & 0x7FFFFFFFu);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && m) atomicMax(out, m);
}

}  // namespace nvfp4
