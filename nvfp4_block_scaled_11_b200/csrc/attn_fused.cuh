// attn_fused.cuh -- ScaleSearchAttention with the scores kept on chip, on the sm_100a tensor cores.
//
// "Search your block floating-point scales!" (gist.science summary of arXiv 2605.12464),
// ScaleSearchAttention > native NVFP4 execution: Q K^T and P V^T run as NVFP4 products with FP32
// accumulation and the softmax numerators P~ are ScaleSearch-quantized before the second product.  The
// unfused chain writes the FP32 scores to HBM and reads them twice; here they never leave the SM.  The
// 64-key tiles that hold an allowed key of a 128-row query tile are cut into `splits` contiguous ranges so
// that the grid fills every SM whatever the number of query tiles, and four kernels run in turn:
//   expand:      Q, K and V^T written once as FP16 tiles in the MMA's shared-memory layout, so that every
//                later tile is one bulk copy;
//   row maxima:  per range ((splits + 1) / 2 of them), S = alpha g_q g_k (Q K^T) into tensor memory (TMEM)
//                over pairs of tiles and the maximum over each row's allowed keys, written per range;
//   numerators:  per range (two per CTA, one per 512-thread half), S again tile by tile, m = the maximum
//                over all keys, P~ = exp(S - m) (the same exp method as the oracle), ScaleSearch of every
//                16-key block with the tensor scale fl(1/2688) (the library's certified fast score, the
//                definition where it cannot decide), the quantized block written to shared memory as the A
//                operand of O += P~ V^T in TMEM; the range's O accumulator and row sum l are written out
//                (or, with one range, the result);
//   combine:     O = fl(fl(sum of the ranges' accumulators * fl(g_p g_v)) / l), l the sum of the ranges'.
// Every result is the unfused chain's formula: P~'s codes are those of the definition applied to this
// call's own scores, and both products are sums of exact terms accumulated in FP32.
//
// The operands are the library's NVFP4 tensors (codes plus E4M3 scales in the tile layout).  Each 16-element
// block enters the tensor cores as FP16 values v * E4M3(s) without the tensor scale: a product of a
// 2-significant-bit E2M1 value and a 4-bit E4M3 scale lies in [2^-10, 2688] with at most 6 significant bits,
// so it is exact in FP16, and the FP16 tensor-core MMA (kind::f16, FP32 accumulation) forms exactly the
// products the block-scaled FP4 MMA forms.  This keeps scale factors out of TMEM; the quantizer, not the
// tensor pipe, bounds this work.
//
// Layout in shared memory (no swizzle, the MMA's K-major canonical layout): a matrix of R rows and K
// columns of FP16 is stored as 16-byte chunks, chunk c (elements 8c..8c+7) of row r at
//   (r mod 8) * 16 + (r div 8) * SBO + c * 128,   SBO = 128 * K / 8,
// so one MMA instruction (K = 16: chunks 2s and 2s+1) reads from start + 256 s with LBO = 128 and that SBO.
// Two such 64-row tiles one after the other are one 128-row tile of the same layout.
//
// Schedule of the numerator kernel (one barrier per tile and half): S(j) was issued two tiles earlier; a
// thread waits for it, reads its 16 scores, forms and quantizes its block of P~(j), waits for O += P~(j-1)
// V(j-1) (long finished), stores its block of P~(j); after the half's barrier one thread issues O += P~(j)
// V(j) and another S(j + 2).  K(j + 2) is fetched once S(j) has read its buffer, V(j + 1) once O(j - 1) has
// read its buffer.  Kernels that allocate TMEM run one CTA per SM, so each CTA holds two independent halves
// (1024 threads, 64 registers): 192 KB of shared memory and all 512 TMEM columns.
//
// Waits on the MMA and copy completion barriers are bounded; a wait that runs out sets a status word, the
// threads of the CTA leave, the TMEM allocation is released and the outputs are not valid.
#pragma once

#include "attention.cuh"

namespace nvfp4 {

constexpr int kAfBM = 128;         // query rows per CTA (the MMA's M)
constexpr int kAfBN = 64;          // keys per tile (the first MMA's N, the second's K)
constexpr int kAfD = 128;          // head dimension (the first MMA's K, the second's N)
constexpr int kAfThreads = 512;    // a half: 16 warps, 4 per TMEM lane quadrant, one 16-key block each per tile
constexpr int kAfCtaThreads = 2 * kAfThreads;   // two halves, one key range each
constexpr int kAfMaxSplits = 64;   // key ranges per query tile
constexpr int kAfTmemColsMax = 512;   // row-max kernel: four S buffers of 128 columns
constexpr int kAfTmemCols = 512;      // numerator kernel: per half an S double buffer and O (128 columns)

// dynamic shared memory: Q (128 x 128 FP16), then
//   row maxima:  four stages of two K tiles (64 x 128 each);
//   numerators:  per half K tiles x 2, V^T tiles (128 x 64) x 2 and a P~ tile (128 x 64)
constexpr int kAfQBytes = kAfBM * kAfD * 2;
constexpr int kAfKBytes = kAfBN * kAfD * 2;
constexpr int kAfVBytes = kAfD * kAfBN * 2;
constexpr int kAfPBytes = kAfBM * kAfBN * 2;
constexpr int kAfHalfBytes = 2 * kAfKBytes + 2 * kAfVBytes + kAfPBytes;
constexpr int kAfSmemBytes = kAfQBytes + 2 * kAfHalfBytes;

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
  int splits;               // key ranges per query tile
  float* ws_max;            // [max_splits, H * Tq] the row-max kernel's ranges' row maxima
  float* ws_l;              // [splits, H * Tq] the ranges' row sums (splits > 1)
  float* ws_o;              // [splits, H * Tq, D] the ranges' O accumulators (splits > 1)
  int max_splits;           // key ranges per query tile of the row-max kernel ((splits + 1) / 2)
  uint8_t* kx;              // [H, Tk / 64] K tiles in FP16, the MMA's shared-memory layout (16 KB each)
  uint8_t* vx;              // [H, Tk / 64] V^T tiles likewise
  uint8_t* qx;              // [H, Tq / 64] Q tiles likewise (two make a CTA's 128 rows)
  float* out;               // [H, Tq, D]
  float* row_max;           // [H * Tq]
  float* row_sum;           // [H * Tq]
  float* s_out;             // nullable: [H, Tq, Tk] scores (verification)
  uint8_t* p_codes;         // nullable: [H, Tq, Tk/2] P~ codes (verification)
  uint8_t* p_sf;            // nullable: H matrices [Tq, Tk/16] P~ scales, tile layout (verification)
  int* status;              // set to a nonzero value when a wait ran out
};

// The tiles of query tile q0 that hold an allowed key of one of its rows, and range s of them.
__device__ __forceinline__ int af_live_tiles(const AttnFusedParams& a, int64_t q0) {
  const int64_t lim_cta = a.causal ? q0 + kAfBM - 1 + a.q_offset : a.Tk - 1;
  return lim_cta < 0 ? 0 : (int)min(a.Tk / kAfBN, lim_cta / kAfBN + 1);
}
__device__ __forceinline__ void af_range(int live, int s, int ns, int& t0, int& t1) {
  t0 = (int)((int64_t)live * s / ns);
  t1 = (int)((int64_t)live * (s + 1) / ns);
}
// A row's last allowed key, clamped to [-1, Tk - 1].
__device__ __forceinline__ int af_row_limit(const AttnFusedParams& a, int64_t q) {
  return a.causal ? (int)max((int64_t)-1, min(q + a.q_offset, a.Tk - 1)) : (int)(a.Tk - 1);
}

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

// Wait for the phase of parity `parity` of an mbarrier to complete.  Each try suspends the thread until the
// phase completes or kAfWaitHintNs pass (the hint keeps waiting threads from spinning on the barrier, which
// would fill the memory-instruction queue the other warps need); after kAfWaitTries tries (about a second)
// the wait gives up and returns false.
constexpr uint32_t kAfWaitHintNs = 10000;
constexpr uint32_t kAfWaitTries = 100000;
__device__ __forceinline__ bool af_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kAfWaitTries; ++i) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(bar), "r"(parity), "n"(kAfWaitHintNs) : "memory");
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

// 32 consecutive columns of this warp's TMEM lanes in one load (one wait).
__device__ __forceinline__ void af_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
               "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                 "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
                 "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                 "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
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

// A block's codes and scale byte as write_block stores them: 0x7F for a poisoned block, the chosen code
// c0 + fstar, or (no usable code) scale 0 with sign-only zeros.
__device__ __forceinline__ void af_encode_block(const u64 (&x2)[8], bool poisoned, int c0, int fstar,
                                                const CandEntry* tab, uint32_t& wlo, uint32_t& whi,
                                                uint32_t& scale) {
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
  af_encode_block(x2, poisoned, c0, fstar, tab, wlo, whi, scale);
}


constexpr uint32_t kAfSboD = 128 * kAfD / 8;    // tiles whose K is the head dimension (Q, K)
constexpr uint32_t kAfSboN = 128 * kAfBN / 8;   // tiles whose K is a key tile (P~, V^T)
constexpr uint32_t kAfTileBytes = 16384;        // a K tile (64 x 128) or a V^T tile (128 x 64) in FP16

// ---------------------------------------------------------------------------------------------------------
// Q, K and V^T as FP16 tiles in the MMA's shared-memory layout (exact: v * E4M3(s), no tensor scale), once
// per call: kx[h][j] the 64 x 128 K tile j, vx[h][j] the 128 x 64 V^T tile j, qx[h][j] the 64 x 128 Q tile j,
// 16 KB each, so that the kernels below fetch a tile with one bulk copy (two consecutive K or Q tiles form
// one 128-row tile of the same layout).  Grid (max(Tk, Tq) / 64, H, 3), 512 threads: one 16-element block
// each, the eight rows of a core matrix in consecutive threads (128 contiguous bytes per chunk column).
// ---------------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kAfThreads) attn_expand_kernel(const AttnFusedParams a) {
  const int t = threadIdx.x;
  const int64_t j = blockIdx.x, h = blockIdx.y, tiles = a.Tk / kAfBN;
  uint4 lo, hi;
  if (blockIdx.z == 2) {   // Q: 64 rows x 8 blocks, as K
    if (j >= a.Tq / kAfBN) return;
    const int r = (t >> 6) * 8 + (t & 7), kb = (t >> 3) & 7;
    const int64_t row = j * kAfBN + r;
    const uint2 cw = *reinterpret_cast<const uint2*>(a.q_codes + ((h * a.Tq + row) * (kAfD / 16) + kb) * 8);
    af_dequant_block(cw, a.q_sf[af_sf_index(h, row, kb, a.Tq, kAfD / 16)], lo, hi);
    af_store_block(a.qx + (h * (a.Tq / kAfBN) + j) * kAfTileBytes, r, kb, kAfSboD, lo, hi);
    return;
  }
  if (j >= tiles) return;
  if (blockIdx.z == 0) {   // K: 64 keys (8 row groups of 8) x 8 blocks
    const int r = (t >> 6) * 8 + (t & 7), kb = (t >> 3) & 7;
    const int64_t key = j * kAfBN + r;
    const uint2 cw = *reinterpret_cast<const uint2*>(a.k_codes + ((h * a.Tk + key) * (kAfD / 16) + kb) * 8);
    af_dequant_block(cw, a.k_sf[af_sf_index(h, key, kb, a.Tk, kAfD / 16)], lo, hi);
    af_store_block(a.kx + (h * tiles + j) * kAfTileBytes, r, kb, kAfSboD, lo, hi);
  } else {                 // V^T: 128 head-dimension rows (16 row groups of 8) x 4 key blocks
    const int d = (t >> 5) * 8 + (t & 7), kb = (t >> 3) & 3;
    const int64_t c = j * (kAfBN / 16) + kb;
    const uint2 cw = *reinterpret_cast<const uint2*>(a.v_codes + ((h * kAfD + d) * (a.Tk / 16) + c) * 8);
    af_dequant_block(cw, a.v_sf[af_sf_index(h, d, c, kAfD, a.Tk / 16)], lo, hi);
    af_store_block(a.vx + (h * tiles + j) * kAfTileBytes, d, kb, kAfSboN, lo, hi);
  }
}

// One tile (16 KB) from global into shared memory by the bulk-copy engine, its bytes counted on mbarrier
// `bar` (which one thread arms with the byte count in the same call).  Issued by one thread.
__device__ __forceinline__ void af_fetch_tile(uint32_t dst, const uint8_t* src, uint32_t bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "n"(kAfTileBytes) : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "n"(kAfTileBytes), "r"(bar) : "memory");
}

// The CTA's 128 Q rows (two FP16 tiles, 32 KB) by one bulk copy, its bytes counted on `bar`.  One thread.
__device__ __forceinline__ void af_fetch_q(const AttnFusedParams& a, uint32_t dst, int64_t h, int64_t q0, uint32_t bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "n"(2 * kAfTileBytes) : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(a.qx + (h * (a.Tq / kAfBN) + q0 / kAfBN) * kAfTileBytes), "n"(2 * kAfTileBytes),
               "r"(bar) : "memory");
}

// Barrier of one half (named barrier 1 + half, 512 threads); the _or form also returns whether p was set
// in any of its threads.
__device__ __forceinline__ bool af_half_sync_or(int half, bool p) {
  uint32_t r;
  asm volatile("{ .reg .pred a, b; setp.ne.u32 a, %1, 0; bar.red.or.pred b, %2, %3, a; selp.u32 %0, 1, 0, b; }"
               : "=r"(r)
               : "r"((uint32_t)p), "r"(1 + half), "n"(kAfThreads)
               : "memory");
  return r != 0;
}
__device__ __forceinline__ void af_half_sync(int half) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + half), "n"(kAfThreads) : "memory");
}

// S = Q K^T (64 columns of TMEM from tmem_d), completion on bar; issued by one thread.  dq, dk: the
// descriptors of the Q and K tiles (the descriptor of the K step s is the tile's plus 256 s bytes, 16 s in
// the start-address field, which cannot carry out of it below 256 KB of shared memory).
__device__ __forceinline__ void af_issue_s(uint32_t tmem_d, uint64_t dq, uint64_t dk, uint32_t bar) {
  const uint32_t idesc = af_idesc(kAfBN);
#pragma unroll
  for (int s = 0; s < kAfD / 16; ++s) af_mma(tmem_d, dq + 16 * s, dk + 16 * s, idesc, s > 0 ? 1u : 0u);
  af_commit(bar);
}
// O (+)= P~ V^T (128 columns of TMEM from tmem_d), completion on bar; issued by one thread.
__device__ __forceinline__ void af_issue_o(uint32_t tmem_d, uint64_t dp, uint64_t dv, bool acc, uint32_t bar) {
  const uint32_t idesc = af_idesc(kAfD);
#pragma unroll
  for (int s = 0; s < kAfBN / 16; ++s) af_mma(tmem_d, dp + 16 * s, dv + 16 * s, idesc, (acc || s > 0) ? 1u : 0u);
  af_commit(bar);
}

// ---------------------------------------------------------------------------------------------------------
// Row maxima of one key range per CTA: grid (Tq / 128, splits, H), 16 consumer warps and one producer warp.
// The range is walked in pairs of 64-key tiles (two consecutive FP16 tiles form one 128-row tile of the
// same layout): the producer fetches a pair with one bulk copy into one of four K stages and, once it has
// landed and the consumers have released that stage's TMEM buffer, issues S = Q K^T for it (N = 128, or
// 64 for a last single tile) -- the MMA issue blocks the issuing thread for about the MMA's duration, so it
// runs in a warp of its own; the consumers read each S, take the row maxima and release the buffer.
// ---------------------------------------------------------------------------------------------------------
constexpr int kAfMaxPairs = 4;                               // K stages and S buffers (128 columns each)
constexpr int kAfMaxThreads = kAfThreads + 32;
constexpr int kAfMaxSmemBytes = kAfQBytes + kAfMaxPairs * 2 * kAfKBytes;

__global__ void __launch_bounds__(kAfMaxThreads, 1) attn_rowmax_kernel(const AttnFusedParams a) {
  extern __shared__ __align__(1024) uint8_t af_dyn[];
  __shared__ float red[4][kAfBM];
  __shared__ __align__(8) uint64_t bars[3][kAfMaxPairs];   // K landed, S complete, S released
  __shared__ __align__(8) uint64_t bar_q_store;              // Q landed
  __shared__ uint32_t tmem_slot;
  __shared__ int s_fail;

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const bool producer = w == kAfThreads / 32;
  const int qd = w & 3, cb = w >> 2;          // consumers: TMEM lane quadrant; 32-key quarter of a pair
  const int r = 32 * qd + lane;               // consumers: this thread's query row within the CTA
  const int split = blockIdx.y;
  const int64_t h = blockIdx.z, q0 = (int64_t)blockIdx.x * kAfBM, q = q0 + r;
  const int live = af_live_tiles(a, q0);
  int t0, t1;
  af_range(live, split, a.max_splits, t0, t1);
  const int pairs = (t1 - t0 + 1) / 2;
  uint8_t* const sQ = af_dyn;
  uint8_t* const sK0 = af_dyn + kAfQBytes;
  const uint8_t* const kx = a.kx + h * (a.Tk / kAfBN) * kAfTileBytes;
  const uint32_t bar_k0 = af_smem(&bars[0][0]), bar_s0 = af_smem(&bars[1][0]), bar_f0 = af_smem(&bars[2][0]);
  const uint32_t bar_q = af_smem(&bar_q_store);

  if (w == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(af_smem(&tmem_slot)),
                 "r"(kAfTmemColsMax));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // the tiles of pair u: t0 + 2u and, unless it is past the range, t0 + 2u + 1
  auto pair_tiles = [&](int u) { return min(2, t1 - t0 - 2 * u); };
  auto fetch_pair = [&](int u, int i) {
    const uint32_t bytes = (uint32_t)pair_tiles(u) * kAfTileBytes;
    const uint32_t bar = bar_k0 + 8 * i;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(af_smem(sK0) + (uint32_t)i * 2 * kAfKBytes), "l"(kx + (int64_t)(t0 + 2 * u) * kAfTileBytes),
                 "r"(bytes), "r"(bar) : "memory");
  };
  if (producer && lane == 0) {
    for (int i = 0; i < kAfMaxPairs; ++i) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_k0 + 8 * i));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_s0 + 8 * i));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar_f0 + 8 * i), "n"(kAfThreads / 32));
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_q));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (pairs > 0) af_fetch_q(a, af_smem(sQ), h, q0, bar_q);
    for (int u = 0; u < kAfMaxPairs && u < pairs; ++u) fetch_pair(u, u);
    s_fail = 0;
  }
  const float sc_s = __fmul_rn(__fmul_rn(a.alpha, *a.q_g), *a.k_g);
  af_proxy_fence();
  af_fence_before();
  __syncthreads();
  af_fence_after();
  const uint32_t tmem = tmem_slot;
  bool ok = true;

  if (producer) {
    if (lane == 0) {
      const uint64_t dq = af_desc(af_smem(sQ), kAfSboD), dk0 = af_desc(af_smem(sK0), kAfSboD);
      if (pairs > 0) ok = af_wait(bar_q, 0u) && ok;   // Q landed
      for (int u = 0; u < pairs; ++u) {
        const int i = u % kAfMaxPairs;
        const uint32_t par = (uint32_t)(u / kAfMaxPairs) & 1u;
        ok = af_wait(bar_k0 + 8 * i, par) && ok;                               // K pair u landed
        if (u >= kAfMaxPairs) ok = af_wait(bar_f0 + 8 * i, par ^ 1u) && ok;    // S(u - 4) released
        af_fence_after();
        const uint32_t n = (uint32_t)pair_tiles(u) * kAfBN, idesc = af_idesc(n);
        const uint64_t dk = dk0 + (uint64_t)i * (2 * kAfKBytes >> 4);
#pragma unroll
        for (int s = 0; s < kAfD / 16; ++s)
          af_mma(tmem + (uint32_t)i * 2 * kAfBN, dq + 16 * s, dk + 16 * s, idesc, s > 0 ? 1u : 0u);
        af_commit(bar_s0 + 8 * i);
        // the stage of pair u - 1 is free once S(u - 1) has completed: fetch pair u + 3 into it
        if (u >= 1 && u - 1 + kAfMaxPairs < pairs) {
          const int ip = (u - 1) % kAfMaxPairs;
          ok = af_wait(bar_s0 + 8 * ip, (uint32_t)((u - 1) / kAfMaxPairs) & 1u) && ok;
          fetch_pair(u - 1 + kAfMaxPairs, ip);
        }
      }
      if (!ok) s_fail = 1;
    }
  } else {
    const int lim = af_row_limit(a, q);   // this row's last allowed key
    // rounding is monotone: for a positive finite scale c, the largest fl(c s) is fl(c max s), so whole
    // blocks below the row's limit take the maximum of the raw sums (mr) and multiply once at the end
    const bool pos_scale = sc_s > 0.0f && sc_s <= FLT_MAX;
    float m = -INFINITY, mr = -INFINITY;
    for (int u = 0; u < pairs; ++u) {
      const int i = u % kAfMaxPairs;
      ok = af_wait(bar_s0 + 8 * i, (uint32_t)(u / kAfMaxPairs) & 1u) && ok;   // S(u) complete
      af_fence_after();
      const bool mine = 32 * cb < pair_tiles(u) * kAfBN;   // a single last tile has 64 keys
      float s[32];
      if (mine) af_ld32(tmem + ((uint32_t)(32 * qd) << 16) + (uint32_t)i * 2 * kAfBN + 32 * cb, s);
      af_fence_before();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar_f0 + 8 * i) : "memory");
      if (mine) {
        const int rem = lim - ((t0 + 2 * u) * kAfBN + 32 * cb);   // keys at or below the row's limit
        if (pos_scale && rem >= 31) {
#pragma unroll
          for (int k = 0; k < 16; ++k) s[k] = fmaxf(s[k], s[k + 16]);
#pragma unroll
          for (int k = 0; k < 8; ++k) s[k] = fmaxf(s[k], s[k + 8]);
#pragma unroll
          for (int k = 0; k < 4; ++k) s[k] = fmaxf(s[k], s[k + 4]);
          mr = fmaxf(mr, fmaxf(fmaxf(s[0], s[2]), fmaxf(s[1], s[3])));
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k <= rem) m = fmaxf(m, __fmul_rn(s[k], sc_s));
        }
      }
    }
    m = fmaxf(m, __fmul_rn(mr, sc_s));
    red[cb][r] = m;
    if (!ok) s_fail = 1;
  }
  __syncthreads();
  const bool failed = s_fail != 0;
  if (!failed && !producer && cb == 0)
    a.ws_max[((int64_t)split * a.H + h) * a.Tq + q] = fmaxf(fmaxf(red[0][r], red[1][r]), fmaxf(red[2][r], red[3][r]));
  if (failed && tid == 0 && a.status) atomicExch(a.status, 1);
  af_fence_before();
  __syncthreads();
  if (w == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kAfTmemColsMax));
}

// ---------------------------------------------------------------------------------------------------------
// Numerators, their quantization and O += P~ V^T over two key ranges per CTA (one per half):
// grid (Tq / 128, ceil(splits / 2), H), 1024 threads.  Per half: K and V^T tiles double-buffered and fetched
// by bulk copies (K(j + 2) once S(j) has read its buffer, V(j + 1) once O(j - 1) has read its buffer), one
// P~ tile written by the threads, S double-buffered and O in TMEM.
// ---------------------------------------------------------------------------------------------------------
template <int NC>
__global__ void __launch_bounds__(kAfCtaThreads, 1) attn_fused_kernel(const AttnFusedParams a) {
  extern __shared__ __align__(1024) uint8_t af_dyn[];
  __shared__ CandEntry tab_store[kTabSize];
  __shared__ float thr[128];
  __shared__ float red[2][4][kAfBM];
  __shared__ __align__(8) uint64_t bars[2][7];   // per half: S 0, S 1, O, K landed 0, 1, V landed 0, 1
  __shared__ __align__(8) uint64_t bar_q_store;   // Q landed
  __shared__ uint32_t tmem_slot;
  CandEntry* tab = tab_store + kTabPad;

  const int tid = threadIdx.x, half = tid / kAfThreads, t = tid % kAfThreads, w = t >> 5, lane = t & 31;
  const int qd = w & 3, cb = w >> 2;          // TMEM lane quadrant; 16-key block of the tile
  const int r = 32 * qd + lane;               // this thread's query row within the CTA
  const int split = 2 * blockIdx.y + half;
  const int64_t h = blockIdx.z, q0 = (int64_t)blockIdx.x * kAfBM, q = q0 + r;
  const int64_t row = h * a.Tq + q, bpr_v = a.Tk / 16;
  const int live = af_live_tiles(a, q0);
  int t0 = 0, t1 = 0;
  if (split < a.splits) af_range(live, split, a.splits, t0, t1);
  uint8_t* const sQ = af_dyn;
  uint8_t* const sK0 = af_dyn + kAfQBytes + half * kAfHalfBytes;
  uint8_t* const sV0 = sK0 + 2 * kAfKBytes;
  uint8_t* const sP = sV0 + 2 * kAfVBytes;
  const uint8_t* const kx = a.kx + h * (a.Tk / kAfBN) * kAfTileBytes;
  const uint8_t* const vx = a.vx + h * (a.Tk / kAfBN) * kAfTileBytes;

  const float gp = __fdiv_rn(1.0f, kTensorDiv);   // P~'s tensor scale: every row's largest numerator is 1
  build_cand_entries(tab, gp);
  build_c0_thresholds(thr, gp);
  const float inv6g = __frcp_rn(__fmul_rn(6.0f, gp));
  if (tid < 32) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(af_smem(&tmem_slot)),
                 "r"(kAfTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  const uint32_t bar_s0 = af_smem(&bars[half][0]), bar_o = af_smem(&bars[half][2]);
  const uint32_t bar_k0 = af_smem(&bars[half][3]), bar_v0 = af_smem(&bars[half][5]);
  const uint32_t sq = af_smem(sQ), sk0 = af_smem(sK0), sv0 = af_smem(sV0), sp = af_smem(sP);
  const uint32_t bar_q = af_smem(&bar_q_store);
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_q));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // fetched when a half has tiles (that half's issuing thread waits for it, so no copy is left in flight)
    bool work = false;
    for (int s = 2 * (int)blockIdx.y; s < min(2 * (int)blockIdx.y + 2, a.splits); ++s) {
      int r0, r1;
      af_range(live, s, a.splits, r0, r1);
      work = work || r0 < r1;
    }
    if (work) af_fetch_q(a, sq, h, q0, bar_q);
  }
  if (t == 0) {
    for (int i = 0; i < 7; ++i) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_s0 + 8 * i));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int i = 0; i < 2 && t0 + i < t1; ++i)
      af_fetch_tile(sk0 + i * kAfKBytes, kx + (int64_t)(t0 + i) * kAfTileBytes, bar_k0 + 8 * i);
    if (t0 < t1) af_fetch_tile(sv0, vx + (int64_t)t0 * kAfTileBytes, bar_v0);
  }
  // the row maximum over all ranges (the row-max kernel's)
  float m = -INFINITY;
  for (int s = 0; s < a.max_splits; ++s) m = fmaxf(m, a.ws_max[(int64_t)s * a.H * a.Tq + row]);
  const float sc_s = __fmul_rn(__fmul_rn(a.alpha, *a.q_g), *a.k_g);
  af_proxy_fence();
  af_fence_before();
  __syncthreads();
  af_fence_after();
  const uint32_t tmem = tmem_slot + (uint32_t)(half * 4 * kAfBN), t_lane = (uint32_t)(32 * qd) << 16;
  // parity bits: bits 0, 1 S buffers and bit 2 O (all threads); bits 3, 4 K landed (thread 32) and 5, 6 V
  // landed (thread 0)
  uint32_t ph = 0;
  bool ok = true;
  const uint64_t dq = af_desc(sq, kAfSboD), dk0 = af_desc(sk0, kAfSboD);
  const uint64_t dv0 = af_desc(sv0, kAfSboN), dp = af_desc(sp, kAfSboN);
  if (t == 32) {   // the S products' thread (the O products': thread 0)
    if (t0 < t1) ok = af_wait(bar_q, 0u) && ok;   // Q landed
    for (int i = 0; i < 2 && t0 + i < t1; ++i) {
      ok = af_wait(bar_k0 + 8 * i, 0u) && ok;
      ph ^= 8u << i;
      af_issue_s(tmem + kAfBN * i, dq, dk0 + i * (kAfKBytes >> 4), bar_s0 + 8 * i);
    }
  }

  const int lim = af_row_limit(a, q);   // this row's last allowed key
  const u64 sc_s2 = pk2(sc_s, sc_s);
  u64 l2 = pk2(0.0f, 0.0f);
  for (int j = t0; j < t1; ++j) {
    const int b = (j - t0) & 1;
    ok = af_wait(bar_s0 + 8 * b, (ph >> b) & 1u) && ok;   // S(j) complete, K buffer b free
    ph ^= 1u << b;
    af_fence_after();
    if (t == 32 && j + 2 < t1) af_fetch_tile(sk0 + b * kAfKBytes, kx + (int64_t)(j + 2) * kAfTileBytes, bar_k0 + 8 * b);
    const uint32_t ts = tmem + t_lane + kAfBN * b + 16 * cb;
    const int k0 = j * kAfBN + 16 * cb;
    float x[16];
    af_ld16(ts, x);
#pragma unroll
    for (int i = 0; i < 16; i += 2) upk2(mul2(pk2(x[i], x[i + 1]), sc_s2), x[i], x[i + 1]);
    if (a.s_out) {
      float* so = a.s_out + row * a.Tk + k0;
#pragma unroll
      for (int i = 0; i < 16; i += 4) *reinterpret_cast<float4*>(so + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
    }
    if (!exp_fast16(m, x)) {   // rare: a numerator below the fast method's range; the scores again, by pairs
      af_ld16(ts, x);
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        float ea = __fsub_rn(__fmul_rn(x[i], sc_s), m), eb = __fsub_rn(__fmul_rn(x[i + 1], sc_s), m);
        exp_ss2(ea, eb);
        x[i] = ea;
        x[i + 1] = eb;
      }
    }
    af_fence_before();
    const int rem = lim - k0;
    if (rem < 15) {
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i > rem) x[i] = 0.0f;
    }
    u64 x2[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      x2[k] = pk2(x[2 * k], x[2 * k + 1]);
      l2 = add2(l2, x2[k]);   // two partial row sums (the sum's order is unspecified)
    }
    uint32_t wlo, whi, scale;
    af_quantize_block<NC>(x2, tab, thr, inv6g, a.f_lo, a.f_hi, wlo, whi, scale);
    if (a.p_codes) {
      *reinterpret_cast<uint2*>(a.p_codes + (row * bpr_v + k0 / 16) * 8) = make_uint2(wlo, whi);
      a.p_sf[af_sf_index(h, q, k0 / 16, a.Tq, bpr_v)] = (uint8_t)scale;
    }
    if (j > t0) {   // O += P~(j-1) V(j-1) complete: the P~ buffer and V buffer b^1 are free
      ok = af_wait(bar_o, (ph >> 2) & 1u) && ok;
      ph ^= 4u;
    }
    if (t == 0 && j + 1 < t1)
      af_fetch_tile(sv0 + (b ^ 1) * kAfVBytes, vx + (int64_t)(j + 1) * kAfTileBytes, bar_v0 + 8 * (b ^ 1));
    {
      uint4 lo, hi;
      af_dequant_block(make_uint2(wlo, whi), scale, lo, hi);
      af_store_block(sP, r, cb, kAfSboN, lo, hi);
    }
    af_proxy_fence();
    af_fence_before();
    if (af_half_sync_or(half, !ok)) {
      ok = false;
      break;
    }
    // the issue of a product holds its thread for about the product's duration: O and S are issued from
    // two warps (thread 0 and thread 32 of the half), so that neither is held back by both
    if (t == 0) {
      ok = af_wait(bar_v0 + 8 * b, (ph >> (5 + b)) & 1u) && ok;   // V(j) landed
      ph ^= 32u << b;
      af_fence_after();
      af_issue_o(tmem + 2 * kAfBN, dp, dv0 + b * (kAfVBytes >> 4), j > t0, bar_o);
    }
    if (t == 32 && j + 2 < t1) {
      ok = af_wait(bar_k0 + 8 * b, (ph >> (3 + b)) & 1u) && ok;   // K(j + 2) landed
      ph ^= 8u << b;
      af_fence_after();
      af_issue_s(tmem + kAfBN * b, dq, dk0 + b * (kAfKBytes >> 4), bar_s0 + 8 * b);
    }
  }
  ok = !af_half_sync_or(half, !ok);   // thread 0's waits after the last barrier included
  if (ok && t1 > t0) {   // the last O += P~ V^T
    ok = af_wait(bar_o, (ph >> 2) & 1u);
    ok = !af_half_sync_or(half, !ok);
    af_fence_after();
  }

  // tiles past every row's last allowed key: P~ is a zero block there (scale 0, zero codes), which is what
  // the verification outputs receive; the products skip those tiles
  if (ok && a.p_codes && split == a.splits - 1) {
    for (int64_t j = live; j < a.Tk / kAfBN; ++j) {
      const int64_t c = j * (kAfBN / 16) + cb;
      *reinterpret_cast<uint2*>(a.p_codes + (row * bpr_v + c) * 8) = make_uint2(0u, 0u);
      a.p_sf[af_sf_index(h, q, c, a.Tq, bpr_v)] = 0;
    }
  }

  // ---- epilogue: the range's O accumulator and row sum, or with one range the result ----
  float l, l_hi;
  upk2(l2, l, l_hi);
  l = __fadd_rn(l, l_hi);
  if (ok && split < a.splits) {
    red[half][cb][r] = l;
    af_half_sync(half);
    l = __fadd_rn(__fadd_rn(__fadd_rn(red[half][0][r], red[half][1][r]), red[half][2][r]), red[half][3][r]);
    const float sc_o = __fmul_rn(gp, *a.v_g);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float o[16];
      if (t1 > t0) {
        af_ld16(tmem + t_lane + 2 * kAfBN + 32 * cb + 16 * hh, o);
      } else {   // no tile in this range: the accumulator is 0
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = 0.0f;
      }
      if (a.splits == 1) {   // with every key in one range: O = fl(fl(acc g_p g_v) / l) (0 / 0 with no key)
        float* op = a.out + row * kAfD + 32 * cb + 16 * hh;
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          *reinterpret_cast<float4*>(op + i) =
              make_float4(__fdiv_rn(__fmul_rn(o[i], sc_o), l), __fdiv_rn(__fmul_rn(o[i + 1], sc_o), l),
                          __fdiv_rn(__fmul_rn(o[i + 2], sc_o), l), __fdiv_rn(__fmul_rn(o[i + 3], sc_o), l));
      } else {
        float* op = a.ws_o + ((int64_t)split * a.H * a.Tq + row) * kAfD + 32 * cb + 16 * hh;
#pragma unroll
        for (int i = 0; i < 16; i += 4) *reinterpret_cast<float4*>(op + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
      }
    }
    if (cb == 0) {
      if (a.splits == 1) {
        a.row_max[row] = m;
        a.row_sum[row] = l;
      } else {
        a.ws_l[(int64_t)split * a.H * a.Tq + row] = l;
      }
    }
  }
  if (!ok && t == 0 && a.status) atomicExch(a.status, 1);
  af_fence_before();
  __syncthreads();
  if (tid < 32) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_slot), "r"(kAfTmemCols));
}

// ---------------------------------------------------------------------------------------------------------
// The ranges combined (splits > 1): a thread per 4 elements of O.
// ---------------------------------------------------------------------------------------------------------
__global__ void attn_combine_kernel(const AttnFusedParams a) {
  const int64_t rows = a.H * a.Tq, i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * (kAfD / 4)) return;
  const int64_t row = i / (kAfD / 4), c4 = i % (kAfD / 4);
  float l = 0.0f, m = -INFINITY;
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int s = 0; s < a.splits; ++s) {
    const int64_t sr = (int64_t)s * rows + row;
    l = __fadd_rn(l, a.ws_l[sr]);
    if (s < a.max_splits) m = fmaxf(m, a.ws_max[sr]);
    const float4 o = *reinterpret_cast<const float4*>(a.ws_o + sr * kAfD + 4 * c4);
    acc = make_float4(__fadd_rn(acc.x, o.x), __fadd_rn(acc.y, o.y), __fadd_rn(acc.z, o.z), __fadd_rn(acc.w, o.w));
  }
  const float sc_o = __fmul_rn(__fdiv_rn(1.0f, kTensorDiv), *a.v_g);
  *reinterpret_cast<float4*>(a.out + row * kAfD + 4 * c4) =
      make_float4(__fdiv_rn(__fmul_rn(acc.x, sc_o), l), __fdiv_rn(__fmul_rn(acc.y, sc_o), l),
                  __fdiv_rn(__fmul_rn(acc.z, sc_o), l), __fdiv_rn(__fmul_rn(acc.w, sc_o), l));
  if (c4 == 0) {
    a.row_max[row] = m;
    a.row_sum[row] = l;
  }
}

}  // namespace nvfp4
