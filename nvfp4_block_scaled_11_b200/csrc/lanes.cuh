// lanes.cuh -- ScaleSearch for small launches: a group of lanes per block, and the batched KV append.
//
// "Search your block floating-point scales!" (gist.science summary of arXiv 2605.12464), Method >
// ScaleSearch, scored exactly as defined (in-order FP32 fold of each candidate's squared errors); the
// launch shape is this library's choice for launches too small to fill the GPU with one block per
// thread (a decode step's KV append, a small batch's activations).
#pragma once

#include "search.cuh"

namespace nvfp4 {

// One block b by a group of G lanes (all G lanes of the group call this together): every lane loads the
// whole block (one transaction per group), derives c0 itself and scores the offsets f_lo + j,
// f_lo + j + G, ... (CPL of them, independent chains) with the definition; the group's smallest
// (SSE, visiting rank) wins, rank 0, 1, 2, 3, ... for f = 0, -1, +1, -2, ..., which is the definition's
// "first strictly smaller SSE in that order".  The lane holding the winner writes the block; when no
// candidate is usable (or the block is zero or poisoned), lane 0 of the group does.  Needs
// f_hi - f_lo < G * CPL.
template <int DT, int MODE, bool ROT, int G, int CPL, bool WANT_SSE, int DEQ>
__device__ __forceinline__ void lanes_block(const QuantParams& p, int64_t b) {
  static_assert(G == 4 || G == 8 || G == 16 || G == 32, "a block group is 4, 8, 16 or 32 lanes");
  const int lane = threadIdx.x & 31, j = lane & (G - 1);
  const unsigned gmask = G == 32 ? 0xFFFFFFFFu : (((1u << G) - 1u) << (lane & ~(G - 1)));
  u64 x2[8];
  load_block_pairs<DT, MODE>(p, b, p.v8 != 0, x2);
  float g = *p.g_src;
  if (p.g_is_amax) g = __fdiv_rn(g, kTensorDiv);
  const bool g_bad = !(g >= 0.0f) || !(g <= FLT_MAX);
  maybe_rotate<ROT>(x2);
  const float amax_b = block_amax_nan(x2);
  const bool poisoned = g_bad || !(amax_b <= FLT_MAX);
  int c0 = 0, fw = -128;
  float rw = 0.0f, sw = 0.0f;
  u64 key = ~0ull;
  if (!poisoned && amax_b != 0.0f) {
    c0 = c0_exact(amax_b, g);
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      // every slot is scored (no branch, so the CPL chains interleave); unusable ones get key ~0
      const int f = p.f_lo + j + G * i, c = c0 + f;
      const bool in = f <= p.f_hi && c >= 1 && c <= 126;
      const float d = in ? __fmul_rn(e4m3_value((uint32_t)c & 0x7Fu), g) : 0.0f;
      const float r = __frcp_rn(d);
      const bool ok = d != 0.0f && fabsf(r) <= FLT_MAX;
      const float s = block_sse_def_pairs(x2, d, ok ? r : 0.0f);   // usable: never NaN (x, v d finite)
      const uint32_t rank = f < 0 ? 2u * (uint32_t)(-f) - 1u : 2u * (uint32_t)f;
      const u64 k = ok ? (((u64)__float_as_uint(s) << 8) | rank) : ~0ull;
      if (k < key) {
        key = k;
        rw = r;
        sw = s;
        fw = f;
      }
    }
  }
  u64 kmin = key;
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) kmin = min(kmin, __shfl_xor_sync(gmask, kmin, o));
  const bool found = kmin != ~0ull;
  if (found ? key == kmin : j == 0)
    write_block<MODE, WANT_SSE, DEQ>(p, b, x2, LaneScales{rw, g}, c0, found ? fw : -128, sw, poisoned, amax_b);
}

// A single launch: block b = thread / G.
template <int DT, int MODE, bool ROT, int G, int CPL, bool WANT_SSE, int DEQ = -1>
__global__ void __launch_bounds__(256) quantize_lanes_kernel(QuantParams p) {
  const int64_t b = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  if (b >= p.nblocks) return;   // whole groups leave together
  lanes_block<DT, MODE, ROT, G, CPL, WANT_SSE, DEQ>(p, b);
}

// Several KV appends in one launch (the K and V groups of every layer of a decode step): item k is a
// KV-append launch's parameters, its blocks numbered start[k] .. start[k + 1] - 1 of the launch.
constexpr int kKvBatchMax = 64;
struct KvBatchParams {
  int count;
  int rot[kKvBatchMax];
  int64_t start[kKvBatchMax + 1];
  QuantParams q[kKvBatchMax];
};
static_assert(sizeof(KvBatchParams) <= 32764, "kernel parameters are limited to 32764 bytes");

template <int G, int CPL>
__global__ void __launch_bounds__(256) kv_append_batch_kernel(const __grid_constant__ KvBatchParams bp) {
  const int64_t b = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  if (b >= bp.start[bp.count]) return;   // whole groups leave together
  int lo = 0, hi = bp.count;             // the item holding b: start[lo] <= b < start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (bp.start[mid] <= b) lo = mid;
    else hi = mid;
  }
  const QuantParams& p = bp.q[lo];
  if (bp.rot[lo]) lanes_block<DT_BF16, SRC_KV, true, G, CPL, false, -1>(p, b - bp.start[lo]);
  else lanes_block<DT_BF16, SRC_KV, false, G, CPL, false, -1>(p, b - bp.start[lo]);
}

}  // namespace nvfp4
