// attn_fused.cuh -- ScaleSearchAttention in one kernel on the sm_100a tensor cores.
//
// "Search your block floating-point scales!" (gist.science summary of arXiv 2605.12464),
// ScaleSearchAttention > native NVFP4 execution: Q K^T and P V^T run as NVFP4 products with FP32
// accumulation and the softmax numerators P~ are ScaleSearch-quantized before the second product.  The
// unfused chain writes the FP32 scores to HBM and reads them twice; here a CTA keeps its 128 query rows'
// scores on chip:
//   sweep 1: for each 64-key tile, S = alpha g_q g_k (Q K^T) into tensor memory (TMEM), row maxima over the
//            allowed keys;
//   sweep 2: S again, P~ = exp(S - m) (the same exp method as the oracle), ScaleSearch of every 16-key
//            block with the tensor scale fl(1/2688) (the library's certified fast score, the definition
//            where it cannot decide), the quantized block written to shared memory as the A operand of
//            O += P~ V^T, accumulated in TMEM;
//   epilogue: O = fl(fl(acc * fl(g_p g_v)) / l), l the FP32 sum of the numerators.
// Every result is the unfused chain's formula: P~'s codes are those of the definition applied to this
// kernel's own scores, and both products are sums of exact terms accumulated in FP32.
//
// The operands are the library's NVFP4 tensors (codes plus E4M3 scales in the tile layout).  Each 16-element
// block is dequantized into shared memory as FP16 values v * E4M3(s) without the tensor scale: a product of
// a 2-significant-bit E2M1 value and a 4-bit E4M3 scale lies in [2^-10, 2688] with at most 6 significant
// bits, so it is exact in FP16, and the FP16 tensor-core MMA (kind::f16, FP32 accumulation) forms exactly
// the products the block-scaled FP4 MMA forms.  This keeps scale factors out of TMEM; the quantizer, not the
// tensor pipe, bounds this kernel.
//
// Layout in shared memory (no swizzle, the MMA's K-major canonical layout): a matrix of R rows and K
// columns of FP16 is stored as 16-byte chunks, chunk c (elements 8c..8c+7) of row r at
//   (r mod 8) * 16 + (r div 8) * SBO + c * 128,   SBO = 128 * K / 8,
// so one MMA instruction (K = 16: chunks 2s and 2s+1) reads from start + 256 s with LBO = 128 and that SBO.
//
// Waits on the MMA completion barriers are bounded; a wait that runs out sets a status word, every thread
// of the CTA leaves, the TMEM allocation is released and the outputs of that CTA are left unwritten.
#pragma once

#include "attention.cuh"

namespace nvfp4 {

constexpr int kAfBM = 128;        // query rows per CTA (the MMA's M)
constexpr int kAfBN = 64;         // keys per tile (the first MMA's N, the second's K)
constexpr int kAfD = 128;         // head dimension (the first MMA's K, the second's N)
constexpr int kAfThreads = 512;   // 16 warps: 4 per TMEM lane quadrant, one 16-key block each per tile
constexpr int kAfTmemCols = 256;  // S double buffer (2 x 64 columns) + O (128 columns)
constexpr uint32_t kAfWaitLimit = 1u << 22;

// dynamic shared memory: Q (128 x 128 FP16), K tiles (64 x 128) x 2, V^T tiles (128 x 64) x 2, P~ (128 x 64) x 2
constexpr int kAfQBytes = kAfBM * kAfD * 2;
constexpr int kAfKBytes = kAfBN * kAfD * 2;
constexpr int kAfVBytes = kAfD * kAfBN * 2;
constexpr int kAfPBytes = kAfBM * kAfBN * 2;
constexpr int kAfSmemBytes = kAfQBytes + 2 * kAfKBytes + 2 * kAfVBytes + 2 * kAfPBytes;

struct AttnFusedParams {
  // operands: codes row-major (16-element blocks along the rows), scales in the tile layout, tensor scale
  const uint8_t* q_codes;   // [H, Tq, D/2]
  const uint8_t* q_sf;      // H matrices [Tq, D/16]
  const float* q_g;
  const uint8_t* k_codes;   // [H, Tk, D/2]
  const uint8_t* k_sf;      // H matrices [Tk, D/16]
  const float* k_g;
  const uint8_t* v_codes;   // V^T: [H, D, Tk/2] (blocks of 16 keys)
  const uint8_t* v_sf;      // H matrices [D, Tk/16]
  const float* v_g;
  int64_t H, Tq, Tk;
  float alpha;
  int causal;               // key k allowed for query q iff k <= q + q_offset
  int64_t q_offset;
  int f_lo, f_hi;
  float* out;               // [H, Tq, D]
  float* row_max;           // [H * Tq]
  float* row_sum;           // [H * Tq]
  float* s_out;             // nullable: [H, Tq, Tk] scores (verification)
  uint8_t* p_codes;         // nullable: [H, Tq, Tk/2] P~ codes (verification)
  uint8_t* p_sf;            // nullable: H matrices [Tq, Tk/16] P~ scales, tile layout (verification)
  int* status;              // set to a nonzero value when a wait ran out
};

__device__ __forceinline__ uint32_t af_smem(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Byte of the tile-layout scale of block column c of row r in matrix `mat` (rows x bpr blocks per matrix).
__device__ __forceinline__ int64_t af_sf_index(int64_t mat, int64_t r, int64_t c, int64_t rows, int64_t bpr) {
  const int64_t ctiles = (bpr + 3) / 4;
  const int64_t mat_bytes = ((rows + 127) / 128) * ctiles * 512;
  return mat * mat_bytes + ((r >> 7) * ctiles + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// One 16-element block (8 code bytes, one scale byte) as 16 FP16 values v * E4M3(s) in two 16-byte chunks.
__device__ __forceinline__ void af_dequant_block(uint2 cw, uint32_t scale, uint4& lo, uint4& hi) {
  uint32_t s2;
  {
    const uint32_t b = (scale & 0xFFu) * 0x0101u;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(s2) : "r"(b));
  }
  uint32_t v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t byte = ((k < 4 ? cw.x : cw.y) >> (8 * (k & 3))) & 0xFFu;
    const uint32_t h2 = e2m1x2_to_f16x2(byte);
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(v[k]) : "r"(h2), "r"(s2));   // exact: see the file comment
  }
  lo = make_uint4(v[0], v[1], v[2], v[3]);
  hi = make_uint4(v[4], v[5], v[6], v[7]);
}

// Store the two chunks of a block at row r, chunks 2 kb and 2 kb + 1, of a canonical K-major tile.
__device__ __forceinline__ void af_store_block(uint8_t* tile, int r, int kb, uint32_t sbo, const uint4& lo,
                                               const uint4& hi) {
  uint8_t* base = tile + (r & 7) * 16 + (r >> 3) * sbo + (2 * kb) * 128;
  *reinterpret_cast<uint4*>(base) = lo;
  *reinterpret_cast<uint4*>(base + 128) = hi;
}

// Matrix descriptor of a canonical K-major tile without swizzle (sm_100 version 1).
__device__ __forceinline__ uint64_t af_desc(uint32_t saddr, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) |
         ((uint64_t)1 << 46);
}

// Instruction descriptor: FP16 A and B, K-major, FP32 accumulator, M = 128, N = n.
__device__ __forceinline__ uint32_t af_idesc(uint32_t n) {
  return (1u << 4) | ((n >> 3) << 17) | ((uint32_t)(kAfBM >> 4) << 24);
}

__device__ __forceinline__ void af_mma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
               "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p; }"
               ::"r"(tmem_d), "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(0u));
}

__device__ __forceinline__ void af_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool af_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kAfWaitLimit; ++i) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    if (ok) return true;
  }
  return false;
}

__device__ __forceinline__ void af_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                 "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void af_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void af_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void af_proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// The definition for the blocks of a warp that the fast score left undecided, one block at a time with the
// whole warp: lane j scores offset f_lo + j of the block (broadcast from its owner), and the smallest
// (SSE, visiting rank) wins -- rank 0, 1, 2, 3, ... for f = 0, -1, +1, -2, ..., which is the definition's
// "first strictly smaller SSE in that order" (the lane-group search's rule).  Called by all 32 lanes.
template <int NC>
__device__ __forceinline__ void af_resolve_deferred(unsigned mask, const u64 (&x2)[8], int c0, int f_lo, int f_hi,
                                                    const CandEntry* tab, int& fstar) {
  const int lane = threadIdx.x & 31;
  while (mask) {
    const int src = __ffs(mask) - 1;
    mask &= mask - 1u;
    float xb[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float lo, hi;
      upk2(x2[k], lo, hi);
      xb[2 * k] = __shfl_sync(0xFFFFFFFFu, lo, src);
      xb[2 * k + 1] = __shfl_sync(0xFFFFFFFFu, hi, src);
    }
    const int cb0 = __shfl_sync(0xFFFFFFFFu, c0, src);
    const int f = f_lo + lane, c = cb0 + f;
    u64 key = ~0ull;
    if (lane < NC && f <= f_hi && c >= 1 && c <= 126) {
      const CandEntry e = tab[c];
      if (e.r != 0.0f) {
        const float sse = block_sse_def(xb, e.d, e.r);
        const uint32_t rank = f < 0 ? 2u * (uint32_t)(-f) - 1u : 2u * (uint32_t)f;
        key = ((u64)__float_as_uint(sse) << 8) | rank;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) key = min(key, __shfl_xor_sync(0xFFFFFFFFu, key, o));
    if (lane == src) {
      if (key == ~0ull) {
        fstar = -128;
      } else {
        const uint32_t rank = (uint32_t)(key & 0xFFu);
        fstar = (rank & 1u) ? -(int)((rank + 1u) >> 1) : (int)(rank >> 1);
      }
    }
  }
}

// One P~ block per lane: ScaleSearch with the tensor scale of the table (each lane's codes, scale byte, as
// write_block would store them), without writing anything.  Called by all 32 lanes of a warp.
template <int NC>
__device__ __forceinline__ void af_quantize_block(const u64 (&x2)[8], const CandEntry* tab, const float* thr,
                                                  float inv6g, int f_lo, int f_hi, uint32_t& wlo, uint32_t& whi,
                                                  uint32_t& scale) {
  const float amax_b = block_amax_nan(x2);
  const bool poisoned = !(amax_b <= FLT_MAX);
  int c0 = 0, fstar = -128;
  float best = 0.0f;
  bool deferred = false;
  if (!poisoned && amax_b != 0.0f) {
    c0 = c0_from_thresholds(thr, amax_b, inv6g);
    if (NC == 1) {
      const int c = c0 + f_lo;
      if (c >= 1 && c <= 126 && tab[c].r != 0.0f) fstar = f_lo;
    } else {
      deferred = !search_fast<NC, false>(x2, amax_b, c0, f_lo, tab, fstar, best);
    }
  }
  if constexpr (NC > 1) {
    const unsigned dm = __ballot_sync(0xFFFFFFFFu, deferred);
    if (dm) af_resolve_deferred<NC>(dm, x2, c0, f_lo, f_hi, tab, fstar);
  }
  wlo = whi = 0u;
  if (poisoned) {
    scale = 0x7Fu;
  } else if (fstar != -128) {
    scale = (uint32_t)(c0 + fstar);
    encode_pairs(x2, tab[scale].r, wlo, whi);
  } else {
    scale = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float lo, hi;
      upk2(x2[k], lo, hi);
      const uint32_t nib = ((__float_as_uint(lo) >> 31) << 3) | ((__float_as_uint(hi) >> 31) << 7);
      if (k < 4) wlo |= nib << (8 * k);
      else whi |= nib << (8 * (k - 4));
    }
  }
}

template <int NC>
__global__ void __launch_bounds__(kAfThreads, 1) attn_fused_kernel(const AttnFusedParams a) {
  extern __shared__ __align__(1024) uint8_t af_dyn[];
  __shared__ CandEntry tab_store[kTabSize];
  __shared__ float thr[128];
  __shared__ float red[4][kAfBM];
  __shared__ __align__(8) uint64_t bars[3];   // S buffer 0, S buffer 1, O
  __shared__ uint32_t tmem_slot;
  __shared__ int s_err;
  CandEntry* tab = tab_store + kTabPad;
  uint8_t* const sQ = af_dyn;
  auto sK = [&](int b) { return af_dyn + kAfQBytes + b * kAfKBytes; };
  auto sV = [&](int b) { return af_dyn + kAfQBytes + 2 * kAfKBytes + b * kAfVBytes; };
  auto sP = [&](int b) { return af_dyn + kAfQBytes + 2 * kAfKBytes + 2 * kAfVBytes + b * kAfPBytes; };
  constexpr uint32_t kSboD = 128 * kAfD / 8;    // tiles whose K is the head dimension (Q, K)
  constexpr uint32_t kSboN = 128 * kAfBN / 8;   // tiles whose K is a key tile (P~, V^T)

  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int qd = w & 3, cb = w >> 2;          // TMEM lane quadrant; 16-key block of the tile
  const int r = 32 * qd + lane;               // this thread's query row within the CTA
  const int64_t h = blockIdx.y, q0 = (int64_t)blockIdx.x * kAfBM, q = q0 + r;
  const int64_t bpr_k = kAfD / 16, bpr_v = a.Tk / 16;

  const float gp = __fdiv_rn(1.0f, kTensorDiv);   // P~'s tensor scale: every row's largest numerator is 1
  build_cand_entries(tab, gp);
  build_c0_thresholds(thr, gp);
  const float inv6g = __frcp_rn(__fmul_rn(6.0f, gp));
  if (w == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(af_smem(&tmem_slot)),
                 "r"(kAfTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (t == 0) {
    for (int i = 0; i < 3; ++i) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(af_smem(&bars[i])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_err = 0;
  }
  // the CTA's Q rows (two blocks per thread)
  for (int i = t; i < kAfBM * (kAfD / 16); i += kAfThreads) {
    const int row = i >> 3, kb = i & 7;
    const int64_t qr = q0 + row;
    uint4 lo, hi;
    const uint2 cw = *reinterpret_cast<const uint2*>(a.q_codes + ((h * a.Tq + qr) * bpr_k + kb) * 8);
    af_dequant_block(cw, a.q_sf[af_sf_index(h, qr, kb, a.Tq, bpr_k)], lo, hi);
    af_store_block(sQ, row, kb, kSboD, lo, hi);
  }
  const float sc_s = __fmul_rn(__fmul_rn(a.alpha, *a.q_g), *a.k_g);
  const float sc_o = __fmul_rn(gp, *a.v_g);
  af_proxy_fence();
  af_fence_before();
  __syncthreads();
  af_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t t_lane = (uint32_t)(32 * qd) << 16;
  // one completion barrier per S buffer (up to two products in flight, each buffer's phase tracked on its
  // own) and one for O
  const uint32_t bar_s[2] = {af_smem(&bars[0]), af_smem(&bars[1])}, bar_o = af_smem(&bars[2]);
  uint32_t ph_s[2] = {0u, 0u}, ph_o = 0;

  const int64_t lim = a.causal ? q + a.q_offset : a.Tk - 1;                   // this row's last allowed key
  const int64_t lim_cta = a.causal ? q0 + kAfBM - 1 + a.q_offset : a.Tk - 1;  // the CTA's last
  const int64_t ntiles = a.Tk / kAfBN;
  const int64_t live = lim_cta < 0 ? 0 : min(ntiles, lim_cta / kAfBN + 1);    // tiles with an allowed key

  // K tile j: 64 keys x 8 blocks, one block per thread (fetched into registers ahead of its use, then
  // dequantized into buffer b); a tile past the end fetches nothing
  struct RawBlock {
    uint2 cw;
    uint32_t sf;
  };
  auto fetch_k = [&](int64_t j) {
    RawBlock rb{make_uint2(0u, 0u), 0u};
    if (j < live) {
      const int key = t >> 3, kb = t & 7;
      const int64_t kr = j * kAfBN + key;
      rb.cw = *reinterpret_cast<const uint2*>(a.k_codes + ((h * a.Tk + kr) * bpr_k + kb) * 8);
      rb.sf = a.k_sf[af_sf_index(h, kr, kb, a.Tk, bpr_k)];
    }
    return rb;
  };
  auto store_k = [&](const RawBlock& rb, int b) {
    uint4 lo, hi;
    af_dequant_block(rb.cw, rb.sf, lo, hi);
    af_store_block(sK(b), t >> 3, t & 7, kSboD, lo, hi);
  };
  // V^T tile j: 128 head-dimension rows x 4 key blocks, one block per thread
  auto fetch_v = [&](int64_t j) {
    RawBlock rb{make_uint2(0u, 0u), 0u};
    if (j < live) {
      const int d = t >> 2, kb = t & 3;
      const int64_t c = j * (kAfBN / 16) + kb;
      rb.cw = *reinterpret_cast<const uint2*>(a.v_codes + ((h * kAfD + d) * bpr_v + c) * 8);
      rb.sf = a.v_sf[af_sf_index(h, d, c, kAfD, bpr_v)];
    }
    return rb;
  };
  auto store_v = [&](const RawBlock& rb, int b) {
    uint4 lo, hi;
    af_dequant_block(rb.cw, rb.sf, lo, hi);
    af_store_block(sV(b), t >> 2, t & 3, kSboN, lo, hi);
  };
  // S = Q K_j^T into TMEM columns 64 b .. 64 b + 63 (issued by thread 0, completion on bar_s[b])
  auto mma_s = [&](int b) {
    if (t == 0) {
      af_fence_after();
      const uint32_t idesc = af_idesc(kAfBN);
#pragma unroll
      for (int s = 0; s < kAfD / 16; ++s)
        af_mma(tmem + kAfBN * b, af_desc(af_smem(sQ) + 256 * s, kSboD), af_desc(af_smem(sK(b)) + 256 * s, kSboD),
               idesc, s > 0 ? 1u : 0u);
      af_commit(b ? bar_s[1] : bar_s[0]);
    }
  };
  // every thread waits; a wait that runs out stops the whole CTA (the flag is read after a barrier)
  auto wait_all = [&](uint32_t bar, uint32_t& ph) -> bool {
    const bool ok = af_wait(bar, ph);
    ph ^= 1u;
    if (!ok) s_err = 1;
    __syncthreads();
    af_fence_after();
    return s_err == 0;
  };
  // this thread's 16 scores of tile j (buffer b), scaled
  auto scores = [&](int b, float (&s)[16]) {
    af_ld16(tmem + t_lane + kAfBN * b + 16 * cb, s);
#pragma unroll
    for (int i = 0; i < 16; ++i) s[i] = __fmul_rn(s[i], sc_s);
  };

  bool ok = true;
  // ---- sweep 1: row maxima over the allowed keys ----
  // two products in flight: S(j + 1) runs while tile j's scores are read, and S(j + 2) is issued into
  // tile j's buffers as soon as they are read; each K tile is fetched into registers two tiles ahead
  float m = -INFINITY;
  RawBlock kn = fetch_k(0), kn2 = fetch_k(1);
  if (live > 0) {
    store_k(kn, 0);
    if (live > 1) store_k(kn2, 1);
    kn = fetch_k(2);
    kn2 = fetch_k(3);
    af_proxy_fence();
    af_fence_before();
    __syncthreads();
    mma_s(0);
    if (live > 1) mma_s(1);
  }
  for (int64_t j = 0; j < live; ++j) {
    const int b = (int)(j & 1);
    ok = b ? wait_all(bar_s[1], ph_s[1]) : wait_all(bar_s[0], ph_s[0]);   // S(j) complete
    if (!ok) break;
    float s[16];
    scores(b, s);
    const int64_t k0 = j * kAfBN + 16 * cb;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (k0 + i <= lim) m = fmaxf(m, s[i]);
    if (j + 2 < live) {
      store_k(kn, b);                          // K(j + 2) into the buffer S(j) has finished reading
      kn = kn2;
      kn2 = fetch_k(j + 4);
      af_proxy_fence();
      af_fence_before();
      __syncthreads();                         // K(j + 2) visible; every thread has read S(j)
      mma_s(b);
    }
  }
  if (ok) {
    red[cb][r] = m;
    __syncthreads();
    m = fmaxf(fmaxf(red[0][r], red[1][r]), fmaxf(red[2][r], red[3][r]));
    __syncthreads();
  }

  // ---- sweep 2: numerators, their quantization, O += P~ V^T ----
  // software-pipelined: S(j + 1) is formed while tile j's numerators are quantized, O += P~(j) V(j) runs
  // while the next tiles are stored, and the raw K and V blocks are fetched a tile ahead of their store
  float l = 0.0f;
  RawBlock kf = fetch_k(1), vf = fetch_v(1);
  if (ok && live > 0) {
    af_fence_before();
    __syncthreads();          // every thread has read its last S of sweep 1
    store_k(fetch_k(0), 0);
    store_v(fetch_v(0), 0);
    af_proxy_fence();
    af_fence_before();
    __syncthreads();
    mma_s(0);
  }
  for (int64_t j = 0; j < live && ok; ++j) {
    const int b = (int)(j & 1);
    if (j + 1 < live) store_k(kf, b ^ 1);     // that buffer's last reader, S(j - 1), has completed
    if (j > 0) {
      ok = wait_all(bar_o, ph_o);              // O(j - 1) complete: its V and P~ buffers are free
      if (!ok) break;
    }
    if (j + 1 < live) store_v(vf, b ^ 1);
    kf = fetch_k(j + 2);
    vf = fetch_v(j + 2);
    af_proxy_fence();
    af_fence_before();
    ok = b ? wait_all(bar_s[1], ph_s[1]) : wait_all(bar_s[0], ph_s[0]);   // S(j) complete; K(j + 1), V(j + 1) visible
    if (!ok) break;
    if (j + 1 < live) mma_s(b ^ 1);
    float s[16], x[16];
    scores(b, s);
    const int64_t k0 = j * kAfBN + 16 * cb;
    if (a.s_out) {
      float* so = a.s_out + (h * a.Tq + q) * a.Tk + k0;
#pragma unroll
      for (int i = 0; i < 16; i += 4) *reinterpret_cast<float4*>(so + i) = make_float4(s[i], s[i + 1], s[i + 2], s[i + 3]);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = s[i];
    if (!exp_fast16(m, x)) {
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        float ea = __fsub_rn(s[i], m), eb = __fsub_rn(s[i + 1], m);
        exp_ss2(ea, eb);
        x[i] = ea;
        x[i + 1] = eb;
      }
    }
    if (k0 + 15 > lim) {
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (k0 + i > lim) x[i] = 0.0f;
    }
    u64 x2[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      l = __fadd_rn(__fadd_rn(l, x[2 * k]), x[2 * k + 1]);
      x2[k] = pk2(x[2 * k], x[2 * k + 1]);
    }
    uint32_t wlo, whi, scale;
    af_quantize_block<NC>(x2, tab, thr, inv6g, a.f_lo, a.f_hi, wlo, whi, scale);
    if (a.p_codes) {
      *reinterpret_cast<uint2*>(a.p_codes + ((h * a.Tq + q) * bpr_v + k0 / 16) * 8) = make_uint2(wlo, whi);
      a.p_sf[af_sf_index(h, q, k0 / 16, a.Tq, bpr_v)] = (uint8_t)scale;
    }
    uint4 lo, hi;
    af_dequant_block(make_uint2(wlo, whi), scale, lo, hi);
    af_store_block(sP(b), r, cb, kSboN, lo, hi);
    af_proxy_fence();
    af_fence_before();
    __syncthreads();
    if (t == 0) {
      af_fence_after();
      const uint32_t idesc = af_idesc(kAfD);
#pragma unroll
      for (int s2 = 0; s2 < kAfBN / 16; ++s2)
        af_mma(tmem + 2 * kAfBN, af_desc(af_smem(sP(b)) + 256 * s2, kSboN), af_desc(af_smem(sV(b)) + 256 * s2, kSboN),
               idesc, (j > 0 || s2 > 0) ? 1u : 0u);
      af_commit(bar_o);
    }
  }
  if (ok && live > 0) ok = wait_all(bar_o, ph_o);   // the last O += P~ V^T

  // tiles past every row's last allowed key: P~ is a zero block there (scale 0, zero codes), which is what
  // the verification outputs receive; the products skip those tiles
  if (ok && a.p_codes) {
    for (int64_t j = live; j < ntiles; ++j) {
      const int64_t c = j * (kAfBN / 16) + cb;
      *reinterpret_cast<uint2*>(a.p_codes + ((h * a.Tq + q) * bpr_v + c) * 8) = make_uint2(0u, 0u);
      a.p_sf[af_sf_index(h, q, c, a.Tq, bpr_v)] = 0;
    }
  }

  // ---- epilogue ----
  if (ok) {
    red[cb][r] = l;
    __syncthreads();
    l = __fadd_rn(__fadd_rn(__fadd_rn(red[0][r], red[1][r]), red[2][r]), red[3][r]);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float o[16];
      if (live > 0) {
        af_ld16(tmem + t_lane + 2 * kAfBN + 32 * cb + 16 * half, o);
      } else {   // no key allowed for any row: the product is 0 (and 0 / 0 is what the chain gives)
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = 0.0f;
      }
      float* op = a.out + (h * a.Tq + q) * kAfD + 32 * cb + 16 * half;
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        *reinterpret_cast<float4*>(op + i) =
            make_float4(__fdiv_rn(__fmul_rn(o[i], sc_o), l), __fdiv_rn(__fmul_rn(o[i + 1], sc_o), l),
                        __fdiv_rn(__fmul_rn(o[i + 2], sc_o), l), __fdiv_rn(__fmul_rn(o[i + 3], sc_o), l));
    }
    if (cb == 0) {
      a.row_max[h * a.Tq + q] = m;
      a.row_sum[h * a.Tq + q] = l;
    }
  } else if (t == 0 && a.status) {
    atomicExch(a.status, 1);
  }
  af_fence_before();
  __syncthreads();
  if (w == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kAfTmemCols));
}

}  // namespace nvfp4
