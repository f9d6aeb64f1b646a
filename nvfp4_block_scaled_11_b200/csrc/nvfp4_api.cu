// nvfp4_api.cu -- the libnvfp4 C ABI (include/nvfp4.h): argument validation and kernel launches.
#include <cuda_runtime.h>
#include <limits.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <initializer_list>
#include <mutex>

#include "../../include/nvfp4.h"
#include "attention.cuh"
#include "attn_fused.cuh"
#include "lanes.cuh"
#include "msda.cuh"
#include "search.cuh"

using namespace nvfp4;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int sms = 0;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_dev[dev].sms == 0) {
    int s = 0;
    cudaDeviceGetAttribute(&s, cudaDevAttrMultiProcessorCount, dev);
    g_dev[dev].sms = s > 0 ? s : 148;
  }
  return g_dev[dev].sms;
}

// Persistent-style grid: enough CTAs for `items` at `per_cta` items each, capped at `ctas_per_sm` per SM.
int grid_for(int64_t items, int per_cta, int ctas_per_sm) {
  int64_t need = (items + per_cta - 1) / per_cta;
  int64_t cap = (int64_t)sm_count() * ctas_per_sm;
  if (need < 1) need = 1;
  return (int)(need < cap ? need : cap);
}

bool checked_mode() {
  static int mode = -1;
  if (mode < 0) {
    const char* e = getenv("NVFP4_CHECKED");
    mode = (e && e[0] == '1') ? 1 : 0;
  }
  return mode == 1;
}

// Host-side fault injection for tests of the CUDA error path: with NVFP4_FAULT_INJECT=launch in the
// environment, nvfp4_dequantize(_ex) asks for blocks of 2048 threads, a configuration the CUDA runtime
// rejects on the host (cudaErrorInvalidConfiguration, nothing reaches the GPU), so the call returns
// NVFP4_ERR_CUDA and the context stays usable.
bool inject_launch_fault() {
  static int mode = -1;
  if (mode < 0) {
    const char* e = getenv("NVFP4_FAULT_INJECT");
    mode = (e && strcmp(e, "launch") == 0) ? 1 : 0;
  }
  return mode == 1;
}

// Largest element count of a one-dimensional call: byte offsets of any element type stay far from
// int64 overflow.
constexpr int64_t kMaxElems = int64_t(1) << 60;

// Product of sizes that must each be non-negative, or -1 when one is negative or the product does not
// fit in int64 (so that no later size arithmetic can wrap round and pass a check).
int64_t checked_prod(std::initializer_list<int64_t> v) {
  int64_t p = 1;
  for (int64_t a : v) {
    if (a < 0 || __builtin_mul_overflow(p, a, &p)) return -1;
  }
  return p;
}

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
inline bool dtype_ok(int dt) { return dt == DT_F32 || dt == DT_BF16 || dt == DT_F16; }
inline int esize(int dt) { return dt == DT_F32 ? 4 : 2; }

int last_error() { return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

int check_finite_sync(const float* g_dev, cudaStream_t s) {
  if (!checked_mode() || g_dev == nullptr) return NVFP4_OK;
  float g = 0.0f;
  if (cudaMemcpyAsync(&g, g_dev, sizeof(float), cudaMemcpyDeviceToHost, s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
  return (g == g && g <= 3.402823466e38f) ? NVFP4_OK : NVFP4_ERR_NONFINITE;
}

int launch_amax(const void* x, int64_t n, int dtype, uint32_t* word, cudaStream_t s) {
  const int64_t vecs = n * esize(dtype) / 32;
  const int grid = grid_for(vecs > 0 ? vecs : 1, 512 * 4, 2);
  const int v8 = aligned(x, 32) ? 1 : 0;
  const char* xp = static_cast<const char*>(x);
  switch (dtype) {
    case DT_F32: amax_kernel<DT_F32><<<grid, 512, 0, s>>>(xp, n, v8, word); break;
    case DT_BF16: amax_kernel<DT_BF16><<<grid, 512, 0, s>>>(xp, n, v8, word); break;
    default: amax_kernel<DT_F16><<<grid, 512, 0, s>>>(xp, n, v8, word); break;
  }
  return last_error();
}

template <int DT, int MODE, bool ROT, int NC>
void launch_search(const QuantParams& p, cudaStream_t s) {
  const int grid = grid_for(p.nblocks, 256, NVFP4_SEARCH_CTAS_PER_SM);
  if constexpr ((MODE == SRC_LINEAR && !ROT) || MODE == SRC_KV) {
    if (p.deq_out) {  // fused round trip: the dequantized values in the input's dtype
      quantize_search_kernel<DT, MODE, ROT, NC, false, DT><<<grid, 256, 0, s>>>(p);
      return;
    }
  }
  if (p.block_sse) quantize_search_kernel<DT, MODE, ROT, NC, true><<<grid, 256, 0, s>>>(p);
  else quantize_search_kernel<DT, MODE, ROT, NC, false><<<grid, 256, 0, s>>>(p);
}

// Launch shapes of the search (windows of at most 32 offsets; wider ones always take a thread per block),
// chosen by the threads a lane-group launch would start (blocks x lanes per block): up to g_lane1_max,
// a half warp / warp per block with one offset per lane (shortest chain); up to g_lanes_max, 4 / 8
// lanes per block with 3 / 4 offsets each (fewer instructions per block); beyond, a thread per block
// with the certified fast score.  Defaults: the crossovers measured on B200, which fall at about the
// same thread counts for both group sizes of a shape.
constexpr int64_t kLane1DefaultMax = 65536;
constexpr int64_t kLanesDefaultMax = 393216;
std::atomic<int64_t> g_lane1_max{kLane1DefaultMax};
std::atomic<int64_t> g_lanes_max{kLanesDefaultMax};

template <int DT, int MODE, bool ROT, int G, int CPL>
void launch_lanes(const QuantParams& p, cudaStream_t s) {
  const int grid = (int)((p.nblocks * G + 255) / 256);
  if constexpr ((MODE == SRC_LINEAR && !ROT) || MODE == SRC_KV) {
    if (p.deq_out) {
      quantize_lanes_kernel<DT, MODE, ROT, G, CPL, false, DT><<<grid, 256, 0, s>>>(p);
      return;
    }
  }
  if (p.block_sse) quantize_lanes_kernel<DT, MODE, ROT, G, CPL, true><<<grid, 256, 0, s>>>(p);
  else quantize_lanes_kernel<DT, MODE, ROT, G, CPL, false><<<grid, 256, 0, s>>>(p);
}

template <int DT, int MODE, bool ROT>
void launch_quantize_dt(const QuantParams& p, cudaStream_t s) {
  const int nc = p.f_hi - p.f_lo + 1;
  if (nc <= 32) {   // nblocks < 2^56, so the thread counts fit in int64
    if (p.nblocks * (nc <= 16 ? 16 : 32) <= g_lane1_max.load(std::memory_order_relaxed)) {
      if (nc <= 16) launch_lanes<DT, MODE, ROT, 16, 1>(p, s);
      else launch_lanes<DT, MODE, ROT, 32, 1>(p, s);
      return;
    }
    if (p.nblocks * (nc <= 12 ? 4 : 8) <= g_lanes_max.load(std::memory_order_relaxed)) {
      if (nc <= 12) launch_lanes<DT, MODE, ROT, 4, 3>(p, s);
      else launch_lanes<DT, MODE, ROT, 8, 4>(p, s);
      return;
    }
  }
  switch (nc) {
    case 1: launch_search<DT, MODE, ROT, 1>(p, s); break;
    case 9: launch_search<DT, MODE, ROT, 9>(p, s); break;
    case 17: launch_search<DT, MODE, ROT, 17>(p, s); break;
    default: quantize_kernel<DT, MODE, ROT><<<grid_for(p.nblocks, 256, 4), 256, 0, s>>>(p); break;
  }
}

// MODE: SRC_LINEAR (any dtype), SRC_KV (BF16 keys), SRC_COLS (any dtype, never rotated).
template <int MODE, bool ROT>
int launch_quantize_t(int dtype, const QuantParams& p, cudaStream_t s) {
  if constexpr (MODE == SRC_KV) {
    launch_quantize_dt<DT_BF16, MODE, ROT>(p, s);
  } else {
    switch (dtype) {
      case DT_F32: launch_quantize_dt<DT_F32, MODE, ROT>(p, s); break;
      case DT_BF16: launch_quantize_dt<DT_BF16, MODE, ROT>(p, s); break;
      default: launch_quantize_dt<DT_F16, MODE, ROT>(p, s); break;
    }
  }
  return last_error();
}

int window_ok(int f_lo, int f_hi) { return f_lo <= f_hi && f_lo >= -126 && f_hi <= 126; }

// Shared body of the quantize entry points; `sf` carries the tile-layout fields (sf.sf_bpr == 0: linear).
int quantize_impl(const void* x, int64_t n, int dtype, int f_lo, int f_hi, const float* gscale_in, uint8_t* codes,
                  uint8_t* scales, float* gscale, int8_t* block_f, float* block_sse, const QuantParams& sf,
                  cudaStream_t s) {
  if (!dtype_ok(dtype) || !window_ok(f_lo, f_hi)) return NVFP4_ERR_ARG;
  if (gscale_in == nullptr && gscale == nullptr) return NVFP4_ERR_ARG;
  if (n < 0 || n % 16 != 0 || n > kMaxElems) return NVFP4_ERR_SIZE;
  if (n > 0 && (x == nullptr || codes == nullptr || scales == nullptr)) return NVFP4_ERR_ARG;
  if ((n > 0 && !aligned(x, 16)) || (n > 0 && !aligned(codes, 8)) || (gscale && !aligned(gscale, 4)) ||
      (gscale_in && !aligned(gscale_in, 4)) || (block_sse && !aligned(block_sse, 4)))
    return NVFP4_ERR_ALIGN;
  QuantParams p{};
  p.x = static_cast<const char*>(x);
  p.nblocks = n / 16;
  p.f_lo = f_lo;
  p.f_hi = f_hi;
  p.codes = codes;
  p.scales = scales;
  p.block_f = block_f;
  p.block_sse = block_sse;
  p.v8 = aligned(x, 32) ? 1 : 0;
  p.sf_bpr = sf.sf_bpr;
  p.sf_rows = sf.sf_rows;
  p.sf_ctiles = sf.sf_ctiles;
  p.sf_mat_bytes = sf.sf_mat_bytes;
  p.tr_cols = sf.tr_cols;
  p.tr_rb = sf.tr_rb;
  p.deq_out = sf.deq_out;
  p.deq_v8 = sf.deq_v8;
  if (gscale_in == nullptr) {
    // gscale doubles as the amax accumulator: zero, reduce, quantize (reads it as amax), then g.
    if (cudaMemsetAsync(gscale, 0, sizeof(float), s) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (n > 0) {
      int rc = launch_amax(x, n, dtype, reinterpret_cast<uint32_t*>(gscale), s);
      if (rc) return rc;
      p.g_src = gscale;
      p.g_is_amax = 1;
      rc = p.tr_cols ? launch_quantize_t<SRC_COLS, false>(dtype, p, s) : launch_quantize_t<SRC_LINEAR, false>(dtype, p, s);
      if (rc) return rc;
    }
    global_scale_kernel<<<1, 32, 0, s>>>(gscale, gscale);
    if (int rc = last_error()) return rc;
    return check_finite_sync(gscale, s);
  }
  p.g_src = gscale_in;
  p.g_is_amax = 0;
  if (n > 0) {
    if (int rc = p.tr_cols ? launch_quantize_t<SRC_COLS, false>(dtype, p, s)
                           : launch_quantize_t<SRC_LINEAR, false>(dtype, p, s))
      return rc;
  }
  if (gscale && gscale != gscale_in) {
    if (cudaMemcpyAsync(gscale, gscale_in, sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return NVFP4_ERR_CUDA;
  }
  return check_finite_sync(gscale_in, s);
}

// Validation and launch parameters of one KV append (nvfp4_kv_append and each item of the batch call);
// p.nblocks == 0 when there is nothing to do.
int kv_append_params(const void* k_bf16, int64_t BH, int64_t T, int64_t first, int64_t n, int64_t D, int f_lo,
                     int f_hi, const float* gscale, uint8_t* codes, uint8_t* scales, int64_t cap, int64_t t0,
                     int scale_layout, QuantParams& p) {
  if (!window_ok(f_lo, f_hi) || gscale == nullptr || (scale_layout != 0 && scale_layout != 1)) return NVFP4_ERR_ARG;
  if (BH < 0 || T < 0 || n < 0 || first < 0 || t0 < 0 || cap < 0 || D <= 0 || D % 16 != 0) return NVFP4_ERR_SIZE;
  if (first > T - n || t0 > cap - n) return NVFP4_ERR_SIZE;
  if (checked_prod({BH, T, D}) < 0 || checked_prod({BH, cap, D}) < 0) return NVFP4_ERR_SIZE;
  if (scale_layout == 1 && BH * cap * (D / 16) >= (int64_t(1) << 32)) return NVFP4_ERR_SIZE;
  if (BH * n * (D / 16) >= (int64_t(1) << 32)) return NVFP4_ERR_SIZE;  // KV block indices are split in 32 bits
  p = QuantParams{};
  if (BH == 0 || n == 0) return NVFP4_OK;
  if (k_bf16 == nullptr || codes == nullptr || scales == nullptr) return NVFP4_ERR_ARG;
  if (!aligned(k_bf16, 16) || !aligned(codes, 8) || !aligned(gscale, 4)) return NVFP4_ERR_ALIGN;
  p.x = static_cast<const char*>(k_bf16);
  p.nblocks = BH * n * (D / 16);
  p.f_lo = f_lo;
  p.f_hi = f_hi;
  p.g_src = gscale;
  p.g_is_amax = 0;
  p.codes = codes;
  p.scales = scales;
  p.v8 = aligned(k_bf16, 32) ? 1 : 0;
  p.T = T;
  p.Tm = n;
  p.sink = first;
  p.D = D;
  p.bpr = D / 16;
  p.out_cap = cap;
  p.out_t0 = t0;
  if (scale_layout == 1) {
    p.sf_bpr = (uint32_t)(D / 16);
    p.sf_rows = (uint32_t)cap;
    p.sf_ctiles = (uint32_t)((D / 16 + 3) / 4);
    p.sf_mat_bytes = ((cap + 127) / 128) * 128 * (int64_t)p.sf_ctiles * 4;
  }
  return NVFP4_OK;
}

// Validation shared by the two deformable-attention entry points; fills the level fields of p.
int msda_setup(MsdaParams& p, int64_t bs, int64_t nkeys, int64_t heads, int64_t ch, const int64_t* shapes, int L, int P,
               int64_t nq, const float* loc, const float* w, float* out) {
  if (L < 1 || L > kMsdaMaxLevels || P < 1 || shapes == nullptr) return NVFP4_ERR_ARG;
  if (bs < 0 || nkeys < 0 || heads < 0 || nq < 0 || (ch != 16 && ch != 32 && ch != 64)) return NVFP4_ERR_SIZE;
  int64_t keys = 0;
  for (int l = 0; l < L; ++l) {
    const int64_t H = shapes[2 * l], W = shapes[2 * l + 1];
    if (H < 1 || W < 1 || H >= (1 << 24) || W >= (1 << 24)) return NVFP4_ERR_SIZE;
    p.H[l] = (int)H;
    p.W[l] = (int)W;
    p.start[l] = keys;
    keys += H * W;
  }
  if (keys != nkeys) return NVFP4_ERR_SIZE;
  if (checked_prod({bs, nkeys, heads, ch}) < 0 || checked_prod({bs, nq, heads, (int64_t)L, (int64_t)P, 2}) < 0 ||
      checked_prod({bs, nq, heads, ch}) < 0)
    return NVFP4_ERR_SIZE;
  p.nkeys = nkeys;
  p.heads = heads;
  p.nq = nq;
  p.total = bs * nq * heads;
  p.L = L;
  p.P = P;
  p.loc = loc;
  p.w = w;
  p.out = out;
  if (p.total == 0) return NVFP4_OK;
  if (loc == nullptr || w == nullptr || out == nullptr) return NVFP4_ERR_ARG;
  if (!aligned(loc, 4) || !aligned(w, 4) || !aligned(out, 32)) return NVFP4_ERR_ALIGN;
  return NVFP4_OK;
}

// Channels per thread: NVFP4 values keep a whole head per thread (its gathers are 8-16 bytes, so the
// per-point location work dominates); full-precision twins split a head into 16-channel slices (their
// gathers are 32-64 bytes per slice, and more threads in flight hide them better).  Both measured.
template <int VT, int CH>
void msda_launch_ch(const MsdaParams& p, cudaStream_t s) {
  constexpr int SPLIT = VT == MSDA_NVFP4 ? 1 : CH / 16;
  msda_forward_kernel<VT, CH, SPLIT><<<grid_for(p.total * SPLIT, 128, 16), 128, 0, s>>>(p);
}

template <int VT>
int msda_launch(const MsdaParams& p, int64_t ch, cudaStream_t s) {
  if (ch == 16) msda_launch_ch<VT, 16>(p, s);
  else if (ch == 32) msda_launch_ch<VT, 32>(p, s);
  else msda_launch_ch<VT, 64>(p, s);
  return last_error();
}

}  // namespace

extern "C" {

const char* nvfp4_status_str(int status) {
  switch (status) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_ARG: return "NVFP4_ERR_ARG: invalid argument";
    case NVFP4_ERR_SIZE: return "NVFP4_ERR_SIZE: size is not a whole number of 16-element blocks";
    case NVFP4_ERR_ALIGN: return "NVFP4_ERR_ALIGN: buffer misaligned";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA: CUDA error";
    case NVFP4_ERR_NONFINITE: return "NVFP4_ERR_NONFINITE: input held NaN or Inf";
    default: return "NVFP4: unknown status";
  }
}

int nvfp4_version(void) { return 100; }

int nvfp4_search_policy(int64_t lane1_max, int64_t lanes_max, int64_t* old_lane1_max, int64_t* old_lanes_max) {
  if (lane1_max < -1 || lanes_max < -1) return NVFP4_ERR_ARG;
  const int64_t a = lane1_max == -1 ? g_lane1_max.load() : g_lane1_max.exchange(lane1_max);
  const int64_t b = lanes_max == -1 ? g_lanes_max.load() : g_lanes_max.exchange(lanes_max);
  if (old_lane1_max) *old_lane1_max = a;
  if (old_lanes_max) *old_lanes_max = b;
  return NVFP4_OK;
}

int nvfp4_tensor_amax(const void* x, int64_t n, int dtype, float* d_amax, void* stream) {
  if (!dtype_ok(dtype) || d_amax == nullptr || (n > 0 && x == nullptr)) return NVFP4_ERR_ARG;
  if (n < 0 || n > kMaxElems) return NVFP4_ERR_SIZE;
  if ((n > 0 && !aligned(x, 16)) || !aligned(d_amax, 4)) return NVFP4_ERR_ALIGN;
  cudaStream_t s = S(stream);
  if (cudaMemsetAsync(d_amax, 0, sizeof(float), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (n == 0) return NVFP4_OK;
  return launch_amax(x, n, dtype, reinterpret_cast<uint32_t*>(d_amax), s);
}

int nvfp4_global_scale(const float* d_amax, float* d_gscale, void* stream) {
  if (d_amax == nullptr || d_gscale == nullptr) return NVFP4_ERR_ARG;
  if (!aligned(d_amax, 4) || !aligned(d_gscale, 4)) return NVFP4_ERR_ALIGN;
  global_scale_kernel<<<1, 32, 0, S(stream)>>>(d_amax, d_gscale);
  return last_error();
}

int nvfp4_quantize_ex(const void* x, int64_t n, int dtype, int block, int f_lo, int f_hi, const float* gscale_in,
                      uint8_t* codes, uint8_t* scales, float* gscale, int8_t* block_f, float* block_sse,
                      void* stream) {
  if (block != 16) return NVFP4_ERR_ARG;
  return quantize_impl(x, n, dtype, f_lo, f_hi, gscale_in, codes, scales, gscale, block_f, block_sse, QuantParams{},
                       S(stream));
}

int64_t nvfp4_sf_mma_bytes(int64_t rows, int64_t cols, int64_t batch) {
  if (rows < 0 || cols < 0 || batch < 0) return NVFP4_ERR_ARG;
  if (cols % 16 != 0) return NVFP4_ERR_SIZE;
  const int64_t b = checked_prod({batch, (rows + 127) / 128, 128, (cols / 16 + 3) / 4, 4});
  return b < 0 ? NVFP4_ERR_SIZE : b;
}

int nvfp4_quantize_mma(const void* x, int64_t batch, int64_t rows, int64_t cols, int dtype, int f_lo, int f_hi,
                       const float* gscale_in, uint8_t* codes, uint8_t* sf, float* gscale, void* stream) {
  if (batch < 0 || rows < 0 || cols < 0) return NVFP4_ERR_ARG;
  if (cols % 16 != 0) return NVFP4_ERR_SIZE;
  const int64_t n = checked_prod({batch, rows, cols});
  if (n < 0 || n / 16 >= (int64_t(1) << 32)) return NVFP4_ERR_SIZE;
  if (n > 0 && sf == nullptr) return NVFP4_ERR_ARG;
  cudaStream_t s = S(stream);
  QuantParams lay{};
  if (n > 0) {
    const int64_t bpr = cols / 16;
    lay.sf_bpr = (uint32_t)bpr;
    lay.sf_rows = (uint32_t)rows;
    lay.sf_ctiles = (uint32_t)((bpr + 3) / 4);
    lay.sf_mat_bytes = ((rows + 127) / 128) * 128 * (int64_t)lay.sf_ctiles * 4;
    // padding bytes (rows up to a multiple of 128, block columns up to a multiple of 4) must read as 0
    if ((rows % 128 != 0 || bpr % 4 != 0) &&
        cudaMemsetAsync(sf, 0, (size_t)(batch * lay.sf_mat_bytes), s) != cudaSuccess)
      return NVFP4_ERR_CUDA;
  }
  return quantize_impl(x, n, dtype, f_lo, f_hi, gscale_in, codes, sf, gscale, nullptr, nullptr, lay, s);
}

int nvfp4_quantize_mma_t(const void* x, int64_t batch, int64_t rows, int64_t cols, int dtype, int f_lo, int f_hi,
                         const float* gscale_in, uint8_t* codes_t, uint8_t* sf_t, float* gscale, void* stream) {
  if (batch < 0 || rows < 0 || cols < 0) return NVFP4_ERR_ARG;
  if (rows % 16 != 0) return NVFP4_ERR_SIZE;
  const int64_t n = checked_prod({batch, rows, cols});
  if (n < 0 || n / 16 >= (int64_t(1) << 32)) return NVFP4_ERR_SIZE;
  if (n > 0 && sf_t == nullptr) return NVFP4_ERR_ARG;
  cudaStream_t s = S(stream);
  QuantParams lay{};
  if (n > 0) {
    const int64_t bpr = rows / 16;           // blocks per row of the transposed [cols, rows] matrix
    lay.sf_bpr = (uint32_t)bpr;
    lay.sf_rows = (uint32_t)cols;
    lay.sf_ctiles = (uint32_t)((bpr + 3) / 4);
    lay.sf_mat_bytes = ((cols + 127) / 128) * 128 * (int64_t)lay.sf_ctiles * 4;
    lay.tr_cols = cols;
    lay.tr_rb = bpr;
    if ((cols % 128 != 0 || bpr % 4 != 0) &&
        cudaMemsetAsync(sf_t, 0, (size_t)(batch * lay.sf_mat_bytes), s) != cudaSuccess)
      return NVFP4_ERR_CUDA;
  }
  return quantize_impl(x, n, dtype, f_lo, f_hi, gscale_in, codes_t, sf_t, gscale, nullptr, nullptr, lay, s);
}

int nvfp4_quantize(const void* x, int64_t n, int dtype, int block, int f_lo, int f_hi, uint8_t* codes,
                   uint8_t* scales, float* gscale, void* stream) {
  if (gscale == nullptr) return NVFP4_ERR_ARG;
  return nvfp4_quantize_ex(x, n, dtype, block, f_lo, f_hi, nullptr, codes, scales, gscale, nullptr, nullptr,
                           stream);
}

int nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* gscale, int64_t n, int out_dtype,
                     void* out, void* stream) {
  return nvfp4_dequantize_ex(codes, scales, gscale, n, out_dtype, out, 0, stream);
}

int nvfp4_quantize_dequantize(const void* x, int64_t n, int dtype, int f_lo, int f_hi, const float* gscale_in,
                              uint8_t* codes, uint8_t* scales, float* gscale, void* out, void* stream) {
  if (!dtype_ok(dtype) || !window_ok(f_lo, f_hi)) return NVFP4_ERR_ARG;
  if (n > 0 && out == nullptr) return NVFP4_ERR_ARG;
  if (n > 0 && !aligned(out, 16)) return NVFP4_ERR_ALIGN;
  const int nc = f_hi - f_lo + 1;
  cudaStream_t s = S(stream);
  if (nc == 1 || nc == 9 || nc == 17) {
    QuantParams sf{};
    sf.deq_out = static_cast<char*>(out);
    sf.deq_v8 = aligned(out, 32) ? 1 : 0;
    return quantize_impl(x, n, dtype, f_lo, f_hi, gscale_in, codes, scales, gscale, nullptr, nullptr, sf, s);
  }
  // other window widths: the two passes, the dequantize reading the codes just written
  QuantParams sf{};
  if (int rc = quantize_impl(x, n, dtype, f_lo, f_hi, gscale_in, codes, scales, gscale, nullptr, nullptr, sf, s))
    return rc;
  return nvfp4_dequantize_ex(codes, scales, gscale_in ? gscale_in : gscale, n, dtype, out, 0, stream);
}

int nvfp4_dequantize_ex(const uint8_t* codes, const uint8_t* scales, const float* gscale, int64_t n, int out_dtype,
                        void* out, int ctas_per_sm, void* stream) {
  if (!dtype_ok(out_dtype) || gscale == nullptr || ctas_per_sm < 0 || ctas_per_sm > 8) return NVFP4_ERR_ARG;
  if (n < 0 || n % 16 != 0 || n > kMaxElems) return NVFP4_ERR_SIZE;
  if (n == 0) return NVFP4_OK;
  if (codes == nullptr || scales == nullptr || out == nullptr) return NVFP4_ERR_ARG;
  if (!aligned(codes, 8) || !aligned(out, 16) || !aligned(gscale, 4)) return NVFP4_ERR_ALIGN;
  const int64_t nb = n / 16;
  const int grid = grid_for(nb, 256, ctas_per_sm ? ctas_per_sm : 8);
  const int v8 = aligned(out, 32) ? 1 : 0;
  char* o = static_cast<char*>(out);
  cudaStream_t s = S(stream);
  const int threads = inject_launch_fault() ? 2048 : 256;
  switch (out_dtype) {
    case DT_F32: dequantize_kernel<DT_F32><<<grid, threads, 0, s>>>(codes, scales, gscale, nb, o, v8); break;
    case DT_BF16: dequantize_kernel<DT_BF16><<<grid, threads, 0, s>>>(codes, scales, gscale, nb, o, v8); break;
    default: dequantize_kernel<DT_F16><<<grid, threads, 0, s>>>(codes, scales, gscale, nb, o, v8); break;
  }
  return last_error();
}

int nvfp4_hadamard16(const void* x, int64_t n, int dtype, void* out, int out_dtype, void* stream) {
  return nvfp4_hadamard16_ex(x, n, dtype, out, out_dtype, 0u, 0, stream);
}

int nvfp4_hadamard16_ex(const void* x, int64_t n, int dtype, void* out, int out_dtype, uint32_t signs,
                        int inverse, void* stream) {
  if (!dtype_ok(dtype) || !dtype_ok(out_dtype) || signs > 0xFFFFu || (inverse != 0 && inverse != 1))
    return NVFP4_ERR_ARG;
  if (n < 0 || n % 16 != 0 || n > kMaxElems) return NVFP4_ERR_SIZE;
  if (n == 0) return NVFP4_OK;
  if (x == nullptr || out == nullptr) return NVFP4_ERR_ARG;
  if (x == out && dtype != out_dtype) return NVFP4_ERR_ARG;
  if (!aligned(x, 16) || !aligned(out, 16)) return NVFP4_ERR_ALIGN;
  const int64_t ng = n / 16;
  const int grid = grid_for(ng, 256, 8);
  const int v8i = aligned(x, 32) ? 1 : 0, v8o = aligned(out, 32) ? 1 : 0;
  const char* xp = static_cast<const char*>(x);
  char* o = static_cast<char*>(out);
  cudaStream_t s = S(stream);
#define NVFP4_H16(DI, DO) hadamard16_kernel<DI, DO><<<grid, 256, 0, s>>>(xp, ng, o, v8i, v8o, signs, inverse)
  if (dtype == DT_F32) {
    if (out_dtype == DT_F32) NVFP4_H16(DT_F32, DT_F32);
    else if (out_dtype == DT_BF16) NVFP4_H16(DT_F32, DT_BF16);
    else NVFP4_H16(DT_F32, DT_F16);
  } else if (dtype == DT_BF16) {
    if (out_dtype == DT_F32) NVFP4_H16(DT_BF16, DT_F32);
    else if (out_dtype == DT_BF16) NVFP4_H16(DT_BF16, DT_BF16);
    else NVFP4_H16(DT_BF16, DT_F16);
  } else {
    if (out_dtype == DT_F32) NVFP4_H16(DT_F16, DT_F32);
    else if (out_dtype == DT_BF16) NVFP4_H16(DT_F16, DT_BF16);
    else NVFP4_H16(DT_F16, DT_F16);
  }
#undef NVFP4_H16
  return last_error();
}

// mid_out (optional, linear scales only): the middle's dequantized values, BF16 [BH, Tm, D] in the
// codes' block order (the rotated values when rotating), written by the search kernel for windows of
// 1, 9 or 17 offsets and by the dequantize kernel otherwise.
static int kv_mixed_impl(const void* k_bf16, int64_t B, int64_t H, int64_t T, int64_t D, int sink_tokens,
                         int recent_tokens, int rotate, int f_lo, int f_hi, void* sink_bf16, void* recent_bf16,
                         uint8_t* codes, uint8_t* scales, float* gscale, bool mma, void* stream,
                         void* mid_out = nullptr) {
  if (!window_ok(f_lo, f_hi) || gscale == nullptr || sink_tokens < 0 || recent_tokens < 0) return NVFP4_ERR_ARG;
  if (B < 0 || H < 0 || T < 0 || D <= 0 || D % 16 != 0 || T < (int64_t)sink_tokens + recent_tokens)
    return NVFP4_ERR_SIZE;
  if (checked_prod({B, H, T, D}) < 0) return NVFP4_ERR_SIZE;
  const int64_t BH = B * H;
  const int64_t Tm = T - sink_tokens - recent_tokens;
  const int64_t ngroups = BH * Tm * (D / 16);
  if (BH > 0 && k_bf16 == nullptr) return NVFP4_ERR_ARG;
  if (BH > 0 && sink_tokens > 0 && sink_bf16 == nullptr) return NVFP4_ERR_ARG;
  if (BH > 0 && recent_tokens > 0 && recent_bf16 == nullptr) return NVFP4_ERR_ARG;
  if (ngroups > 0 && (codes == nullptr || scales == nullptr)) return NVFP4_ERR_ARG;
  if (ngroups >= (int64_t(1) << 32)) return NVFP4_ERR_SIZE;  // KV block indices are split in 32 bits
  if ((BH > 0 && !aligned(k_bf16, 16)) || (sink_bf16 && !aligned(sink_bf16, 16)) ||
      (recent_bf16 && !aligned(recent_bf16, 16)) || (codes && !aligned(codes, 8)) || !aligned(gscale, 4) ||
      (mid_out && !aligned(mid_out, 16)))
    return NVFP4_ERR_ALIGN;
  const int nc = f_hi - f_lo + 1;
  const bool fused = mid_out != nullptr && (nc == 1 || nc == 9 || nc == 17);
  cudaStream_t s = S(stream);
  const char* k = static_cast<const char*>(k_bf16);
  if (BH > 0 && sink_tokens + recent_tokens > 0) {
    const int64_t units = BH * (sink_tokens + recent_tokens) * (D * 2 / 16);
    kv_copy_kernel<<<grid_for(units, 256, 8), 256, 0, s>>>(k, BH, T, D * 2, sink_tokens, recent_tokens,
                                                           static_cast<char*>(sink_bf16),
                                                           static_cast<char*>(recent_bf16));
    if (int rc = last_error()) return rc;
  }
  if (cudaMemsetAsync(gscale, 0, sizeof(float), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (ngroups > 0) {
    const int v8 = aligned(k_bf16, 32) ? 1 : 0;
    const int grid = grid_for(ngroups, 256, 8);
    uint32_t* word = reinterpret_cast<uint32_t*>(gscale);
    if (rotate) kv_amax_kernel<true><<<grid, 256, 0, s>>>(k, ngroups, T, Tm, sink_tokens, D, D / 16, v8, word);
    else kv_amax_kernel<false><<<grid, 256, 0, s>>>(k, ngroups, T, Tm, sink_tokens, D, D / 16, v8, word);
    if (int rc = last_error()) return rc;
    QuantParams p{};
    p.x = k;
    p.nblocks = ngroups;
    p.f_lo = f_lo;
    p.f_hi = f_hi;
    p.g_src = gscale;
    p.g_is_amax = 1;
    p.codes = codes;
    p.scales = scales;
    p.v8 = v8;
    p.T = T;
    p.Tm = Tm;
    p.sink = sink_tokens;
    p.D = D;
    p.bpr = D / 16;
    if (mma) {
      // the scales of each (batch, head) form a [Tm, D/16] matrix in the tensor-core tile layout
      p.sf_bpr = (uint32_t)(D / 16);
      p.sf_rows = (uint32_t)Tm;
      p.sf_ctiles = (uint32_t)((D / 16 + 3) / 4);
      p.sf_mat_bytes = ((Tm + 127) / 128) * 128 * (int64_t)p.sf_ctiles * 4;
      if ((Tm % 128 != 0 || (D / 16) % 4 != 0) &&
          cudaMemsetAsync(scales, 0, (size_t)(BH * p.sf_mat_bytes), s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    }
    if (fused) {
      p.deq_out = static_cast<char*>(mid_out);
      p.deq_v8 = aligned(mid_out, 32) ? 1 : 0;
    }
    int rc = rotate ? launch_quantize_t<SRC_KV, true>(DT_BF16, p, s) : launch_quantize_t<SRC_KV, false>(DT_BF16, p, s);
    if (rc) return rc;
  }
  global_scale_kernel<<<1, 32, 0, s>>>(gscale, gscale);
  if (int rc = last_error()) return rc;
  if (mid_out != nullptr && !fused && ngroups > 0) {
    if (int rc = nvfp4_dequantize_ex(codes, scales, gscale, ngroups * 16, DT_BF16, mid_out, 0, stream)) return rc;
  }
  return check_finite_sync(gscale, s);
}

int nvfp4_msda_forward_nvfp4(const uint8_t* codes, const uint8_t* scales, const float* gscale, int64_t bs,
                             int64_t nkeys, int64_t heads, int64_t ch, const int64_t* shapes, int L, int P, int64_t nq,
                             const float* loc, const float* w, float* out, void* stream) {
  MsdaParams p{};
  if (int rc = msda_setup(p, bs, nkeys, heads, ch, shapes, L, P, nq, loc, w, out)) return rc;
  if (p.total == 0) return NVFP4_OK;
  if (codes == nullptr || scales == nullptr || gscale == nullptr) return NVFP4_ERR_ARG;
  if (!aligned(codes, 16) || !aligned(gscale, 4)) return NVFP4_ERR_ALIGN;
  p.codes = codes;
  p.scales = scales;
  p.gsrc = gscale;
  return msda_launch<MSDA_NVFP4>(p, ch, S(stream));
}

int nvfp4_msda_forward(const void* value, int dtype, int64_t bs, int64_t nkeys, int64_t heads, int64_t ch,
                       const int64_t* shapes, int L, int P, int64_t nq, const float* loc, const float* w, float* out,
                       void* stream) {
  if (!dtype_ok(dtype)) return NVFP4_ERR_ARG;
  MsdaParams p{};
  if (int rc = msda_setup(p, bs, nkeys, heads, ch, shapes, L, P, nq, loc, w, out)) return rc;
  if (p.total == 0) return NVFP4_OK;
  if (value == nullptr) return NVFP4_ERR_ARG;
  if (!aligned(value, 16)) return NVFP4_ERR_ALIGN;
  p.value = static_cast<const char*>(value);
  cudaStream_t s = S(stream);
  if (dtype == DT_F32) return msda_launch<MSDA_F32>(p, ch, s);
  if (dtype == DT_F16) return msda_launch<MSDA_F16>(p, ch, s);
  return msda_launch<MSDA_BF16>(p, ch, s);
}

int nvfp4_softmax_quantize_mma(const float* s, int64_t batch, int64_t Tq, int64_t Tk, int causal, int64_t q_offset,
                               int f_lo, int f_hi, uint8_t* codes, uint8_t* sf, float* gscale, float* row_max,
                               float* row_sum, void* stream) {
  const int nc = f_hi - f_lo + 1;
  if (!window_ok(f_lo, f_hi) || (nc != 1 && nc != 9 && nc != 17) || gscale == nullptr) return NVFP4_ERR_ARG;
  if (batch < 0 || Tq < 0 || Tk < 0 || Tk % 16 != 0) return NVFP4_ERR_SIZE;
  if (checked_prod({batch, Tq, Tk}) < 0) return NVFP4_ERR_SIZE;
  const int64_t rows = batch * Tq, bpr = Tk / 16;
  if (rows * bpr >= (int64_t(1) << 32)) return NVFP4_ERR_SIZE;
  cudaStream_t st = S(stream);
  if (rows == 0 || Tk == 0) return NVFP4_OK;
  if (s == nullptr || codes == nullptr || sf == nullptr || row_max == nullptr || row_sum == nullptr)
    return NVFP4_ERR_ARG;
  if (!aligned(s, 16) || !aligned(codes, 8) || !aligned(gscale, 4) || !aligned(row_max, 4) || !aligned(row_sum, 4))
    return NVFP4_ERR_ALIGN;
  QuantParams p{};
  p.nblocks = rows * bpr;
  p.f_lo = f_lo;
  p.f_hi = f_hi;
  p.codes = codes;
  p.scales = sf;
  p.sf_bpr = (uint32_t)bpr;
  p.sf_rows = (uint32_t)Tq;
  p.sf_ctiles = (uint32_t)((bpr + 3) / 4);
  p.sf_mat_bytes = ((Tq + 127) / 128) * 128 * (int64_t)p.sf_ctiles * 4;
  if ((Tq % 128 != 0 || bpr % 4 != 0) && cudaMemsetAsync(sf, 0, (size_t)(batch * p.sf_mat_bytes), st) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  // warps per row: one while the rows alone give every SM its 32 resident warps (the kernel is bound by
  // instruction issue, and warps that share a row wait for one another twice per row); for fewer, longer
  // rows (decode) up to 8, each warp keeping at least 64 blocks (two rounds of its lanes)
  int wpr = 1;
  while (wpr < 8 && rows * wpr < (int64_t)sm_count() * 32 && bpr >= 128 * (int64_t)wpr) wpr *= 2;
  SoftmaxParams a{s, rows, Tq, Tk, causal ? 1 : 0, q_offset, aligned(s, 32) ? 1 : 0, wpr, row_max, row_sum, gscale};
  const int64_t groups = (rows + 8 / wpr - 1) / (8 / wpr);
  const int grid = grid_for(groups * 256, 256, 4);
#define NVFP4_SOFTMAX(NC) \
  (wpr > 1 ? softmax_quantize_kernel<NC, true><<<grid, 256, 0, st>>>(p, a) \
           : softmax_quantize_kernel<NC, false><<<grid, 256, 0, st>>>(p, a))
  if (nc == 9) NVFP4_SOFTMAX(9);
  else if (nc == 1) NVFP4_SOFTMAX(1);
  else NVFP4_SOFTMAX(17);
#undef NVFP4_SOFTMAX
  return last_error();
}

}  // extern "C"

// The fused attention's kernels raise their shared-memory limit once per device (the attribute belongs to
// the kernel on the current device); one instantiation, so one record, per kernel.
template <auto* kernel>
int af_raise_smem(int bytes) {
  static std::mutex mu;
  static uint64_t done = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> g(mu);
  if ((done >> dev) & 1u) return NVFP4_OK;
  // the largest shared-memory carveout, so that two CTAs of the numerator kernel fit on an SM
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess ||
      cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  done |= 1ull << dev;
  return NVFP4_OK;
}

template <int NC>
int launch_attn_fused(const AttnFusedParams& a, cudaStream_t st) {
  int rc = af_raise_smem<attn_rowmax_kernel>(kAfMaxSmemBytes);
  if (rc == NVFP4_OK) rc = af_raise_smem<attn_fused_kernel<NC>>(kAfSmemBytes);
  if (rc != NVFP4_OK) return rc;
  attn_expand_kernel<<<dim3((unsigned)(std::max(a.Tk, a.Tq) / kAfBN), (unsigned)a.H, 3), kAfThreads, 0, st>>>(a);
  attn_rowmax_kernel<<<dim3((unsigned)(a.Tq / kAfBM), (unsigned)a.max_splits, (unsigned)a.H), kAfMaxThreads,
                       kAfMaxSmemBytes, st>>>(a);
  // a numerator CTA runs two key ranges, one per half
  attn_fused_kernel<NC><<<dim3((unsigned)(a.Tq / kAfBM), (unsigned)((a.splits + 1) / 2), (unsigned)a.H),
                          kAfCtaThreads, kAfSmemBytes, st>>>(a);
  if (a.splits > 1) {
    const int64_t n = a.H * a.Tq * (kAfD / 4);
    attn_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a);
  }
  return last_error();
}

// Workspace: the ranges' O accumulators (splits > 1), row sums (splits > 1) and row maxima, then, from a
// 256-byte boundary, the K, V^T and Q tiles in FP16 (16 KB per 64 keys or query rows and head each).
int64_t af_tiles_offset(int64_t H, int64_t Tq, int64_t splits) {
  const int64_t rows = H * Tq;
  return (splits * rows * 4 + (splits > 1 ? splits * rows * (kAfD + 1) * 4 : 0) + 255) / 256 * 256;
}
size_t af_workspace_bytes(int64_t H, int64_t Tq, int64_t Tk, int64_t splits) {
  return (size_t)(af_tiles_offset(H, Tq, splits) + (2 * H * (Tk / kAfBN) + H * (Tq / kAfBN)) * (int64_t)kAfTileBytes);
}

extern "C" {

size_t nvfp4_attention_fused_workspace_bytes(int64_t H, int64_t Tq, int64_t Tk, int splits) {
  if (H < 0 || Tq < 0 || Tk < 0 || Tk % kAfBN != 0 || splits < 1 || splits > kAfMaxSplits ||
      checked_prod({H, Tq, kAfD + 2, splits, 4}) < 0 || checked_prod({H, Tk + Tq, 2 * kAfD * 2}) < 0)
    return 0;
  return af_workspace_bytes(H, Tq, Tk, splits);
}

int nvfp4_attention_fused_splits(int64_t H, int64_t Tq, int64_t Tk, int* splits) {
  if (!splits) return NVFP4_ERR_ARG;
  if (H < 0 || Tq < 0 || Tk < 0 || Tq % kAfBM != 0 || Tk % kAfBN != 0) return NVFP4_ERR_SIZE;
  *splits = 1;
  const int64_t qt = H * (Tq / kAfBM), tiles = Tk / kAfBN;
  if (qt == 0 || tiles == 0) return NVFP4_OK;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      af_raise_smem<attn_fused_kernel<9>>(kAfSmemBytes) != NVFP4_OK ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_fused_kernel<9>, kAfCtaThreads, kAfSmemBytes) !=
          cudaSuccess)
    return NVFP4_ERR_CUDA;
  const int64_t slots = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
  // waves of equal CTAs, each running two ranges of 1/s of a query tile's keys side by side: s ranges cost
  // ceil(qt ceil(s/2) / slots) / s; ranges of at least 8 tiles; the smallest s within 2 % of the best (fewer
  // ranges to combine)
  const int64_t smax = std::max<int64_t>(1, std::min<int64_t>(kAfMaxSplits, tiles / 8));
  auto cost = [&](int64_t s) { return (double)((qt * ((s + 1) / 2) + slots - 1) / slots) / (double)s; };
  double best = 1e30;
  for (int64_t s = 1; s <= smax; ++s) best = std::min(best, cost(s));
  for (int64_t s = 1; s <= smax; ++s)
    if (cost(s) <= best * 1.02) {
      *splits = (int)s;
      break;
    }
  return NVFP4_OK;
}

int nvfp4_attention_fused(const uint8_t* q_codes, const uint8_t* q_sf, const float* q_gscale, const uint8_t* k_codes,
                          const uint8_t* k_sf, const float* k_gscale, const uint8_t* v_codes_t, const uint8_t* v_sf_t,
                          const float* v_gscale, int64_t H, int64_t Tq, int64_t Tk, int64_t D, float alpha, int causal,
                          int64_t q_offset, int f_lo, int f_hi, int splits, void* workspace, size_t workspace_bytes,
                          float* out, float* row_max, float* row_sum, float* s_out, uint8_t* p_codes, uint8_t* p_sf,
                          int* status, void* stream) {
  const int nc = f_hi - f_lo + 1;
  if (!window_ok(f_lo, f_hi) || (nc != 1 && nc != 9 && nc != 17)) return NVFP4_ERR_ARG;
  if (splits < 1 || splits > kAfMaxSplits) return NVFP4_ERR_ARG;
  if (H < 0 || Tq < 0 || Tk < 0 || D != kAfD || Tq % kAfBM != 0 || Tk % kAfBN != 0) return NVFP4_ERR_SIZE;
  if (H > 65535 || Tk >= ((int64_t)1 << 26) || checked_prod({H, Tq, Tk}) < 0 ||
      checked_prod({H, Tq, D + 2, splits, 4}) < 0)
    return NVFP4_ERR_SIZE;
  if (H == 0 || Tq == 0) return NVFP4_OK;
  if (Tk == 0) return NVFP4_ERR_SIZE;   // no keys: nothing to attend to
  if (!q_codes || !q_sf || !q_gscale || !k_codes || !k_sf || !k_gscale || !v_codes_t || !v_sf_t || !v_gscale ||
      !out || !row_max || !row_sum || !workspace || ((p_codes == nullptr) != (p_sf == nullptr)))
    return NVFP4_ERR_ARG;
  if (checked_prod({H, Tk + Tq, 2 * D * 2}) < 0 || workspace_bytes < af_workspace_bytes(H, Tq, Tk, splits))
    return NVFP4_ERR_SIZE;
  if (!aligned(q_codes, 8) || !aligned(k_codes, 8) || !aligned(v_codes_t, 8) || !aligned(k_sf, 4) || !aligned(out, 16) ||
      !aligned(q_gscale, 4) || !aligned(k_gscale, 4) || !aligned(v_gscale, 4) || !aligned(row_max, 4) ||
      !aligned(row_sum, 4) || !aligned(workspace, 16) || (s_out && !aligned(s_out, 16)) ||
      (p_codes && !aligned(p_codes, 8)) || (status && !aligned(status, 4)))
    return NVFP4_ERR_ALIGN;
  // workspace: the O accumulators first (16-byte aligned rows), then the row sums and the row maxima
  const int64_t rows = H * Tq;
  float* ws = static_cast<float*>(workspace);
  float* ws_o = splits > 1 ? ws : nullptr;
  float* ws_l = splits > 1 ? ws + (int64_t)splits * rows * kAfD : nullptr;
  float* ws_max = splits > 1 ? ws_l + (int64_t)splits * rows : ws;
  uint8_t* kx = static_cast<uint8_t*>(workspace) + af_tiles_offset(H, Tq, splits);
  uint8_t* vx = kx + H * (Tk / kAfBN) * (int64_t)kAfTileBytes;
  uint8_t* qx = vx + H * (Tk / kAfBN) * (int64_t)kAfTileBytes;
  AttnFusedParams a{q_codes, q_sf, q_gscale, k_codes, k_sf, k_gscale, v_codes_t, v_sf_t, v_gscale, H, Tq, Tk,
                    alpha, causal ? 1 : 0, q_offset, f_lo, f_hi, splits, ws_max, ws_l, ws_o, (splits + 1) / 2,
                    kx, vx, qx, out, row_max, row_sum, s_out, p_codes, p_sf, status};
  cudaStream_t st = S(stream);
  if (nc == 9) return launch_attn_fused<9>(a, st);
  if (nc == 1) return launch_attn_fused<1>(a, st);
  return launch_attn_fused<17>(a, st);
}

int nvfp4_rows_divide(float* x, const float* l, int64_t rows, int64_t cols, void* stream) {
  if (rows < 0 || cols < 0 || cols % 4 != 0 || checked_prod({rows, cols}) < 0) return NVFP4_ERR_SIZE;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (x == nullptr || l == nullptr) return NVFP4_ERR_ARG;
  if (!aligned(x, 16) || !aligned(l, 4)) return NVFP4_ERR_ALIGN;
  rows_divide_kernel<<<grid_for(rows * cols / 4, 256, 8), 256, 0, S(stream)>>>(x, l, rows, cols);
  return last_error();
}

int nvfp4_mxfp4_quantize(const void* x, int64_t n, int dtype, uint8_t* codes, uint8_t* scales, void* stream) {
  if (!dtype_ok(dtype)) return NVFP4_ERR_ARG;
  if (n < 0 || n % 32 != 0 || n > kMaxElems) return NVFP4_ERR_SIZE;
  if (n == 0) return NVFP4_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr) return NVFP4_ERR_ARG;
  if (!aligned(x, 16) || !aligned(codes, 16)) return NVFP4_ERR_ALIGN;
  const int64_t nb = n / 32;
  const int grid = grid_for(nb, 256, 8);
  const int v8 = aligned(x, 32) ? 1 : 0;
  const char* xp = static_cast<const char*>(x);
  cudaStream_t s = S(stream);
  switch (dtype) {
    case DT_F32: mxfp4_quantize_kernel<DT_F32><<<grid, 256, 0, s>>>(xp, nb, v8, codes, scales); break;
    case DT_BF16: mxfp4_quantize_kernel<DT_BF16><<<grid, 256, 0, s>>>(xp, nb, v8, codes, scales); break;
    default: mxfp4_quantize_kernel<DT_F16><<<grid, 256, 0, s>>>(xp, nb, v8, codes, scales); break;
  }
  return last_error();
}

int nvfp4_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t n, int out_dtype, void* out,
                           void* stream) {
  if (!dtype_ok(out_dtype)) return NVFP4_ERR_ARG;
  if (n < 0 || n % 32 != 0 || n > kMaxElems) return NVFP4_ERR_SIZE;
  if (n == 0) return NVFP4_OK;
  if (codes == nullptr || scales == nullptr || out == nullptr) return NVFP4_ERR_ARG;
  if (!aligned(codes, 16) || !aligned(out, 16)) return NVFP4_ERR_ALIGN;
  const int64_t nb = n / 32;
  const int grid = grid_for(nb, 256, 8);
  const int v8 = aligned(out, 32) ? 1 : 0;
  char* o = static_cast<char*>(out);
  cudaStream_t s = S(stream);
  switch (out_dtype) {
    case DT_F32: mxfp4_dequantize_kernel<DT_F32><<<grid, 256, 0, s>>>(codes, scales, nb, o, v8); break;
    case DT_BF16: mxfp4_dequantize_kernel<DT_BF16><<<grid, 256, 0, s>>>(codes, scales, nb, o, v8); break;
    default: mxfp4_dequantize_kernel<DT_F16><<<grid, 256, 0, s>>>(codes, scales, nb, o, v8); break;
  }
  return last_error();
}

int nvfp4_kv_gscale(const void* k_bf16, int64_t B, int64_t H, int64_t T, int64_t D, int sink_tokens, int recent_tokens,
                    int rotate, float* gscale, void* stream) {
  if (gscale == nullptr || sink_tokens < 0 || recent_tokens < 0) return NVFP4_ERR_ARG;
  if (B < 0 || H < 0 || T < 0 || D <= 0 || D % 16 != 0 || T < (int64_t)sink_tokens + recent_tokens)
    return NVFP4_ERR_SIZE;
  const int64_t Tm = T - sink_tokens - recent_tokens;
  if (checked_prod({B, H, T, D}) < 0) return NVFP4_ERR_SIZE;
  const int64_t ngroups = B * H * Tm * (D / 16);
  if (ngroups >= (int64_t(1) << 32)) return NVFP4_ERR_SIZE;  // KV block indices are split in 32 bits
  if (ngroups > 0 && k_bf16 == nullptr) return NVFP4_ERR_ARG;
  if ((ngroups > 0 && !aligned(k_bf16, 16)) || !aligned(gscale, 4)) return NVFP4_ERR_ALIGN;
  cudaStream_t s = S(stream);
  if (cudaMemsetAsync(gscale, 0, sizeof(float), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (ngroups > 0) {
    const char* k = static_cast<const char*>(k_bf16);
    const int v8 = aligned(k_bf16, 32) ? 1 : 0;
    const int grid = grid_for(ngroups, 256, 8);
    uint32_t* word = reinterpret_cast<uint32_t*>(gscale);
    if (rotate) kv_amax_kernel<true><<<grid, 256, 0, s>>>(k, ngroups, T, Tm, sink_tokens, D, D / 16, v8, word);
    else kv_amax_kernel<false><<<grid, 256, 0, s>>>(k, ngroups, T, Tm, sink_tokens, D, D / 16, v8, word);
    if (int rc = last_error()) return rc;
  }
  global_scale_kernel<<<1, 32, 0, s>>>(gscale, gscale);
  if (int rc = last_error()) return rc;
  return check_finite_sync(gscale, s);
}

int nvfp4_kv_append(const void* k_bf16, int64_t BH, int64_t T, int64_t first, int64_t n, int64_t D, int rotate,
                    int f_lo, int f_hi, const float* gscale, uint8_t* codes, uint8_t* scales, int64_t cap, int64_t t0,
                    int scale_layout, void* stream) {
  QuantParams p{};
  if (int rc = kv_append_params(k_bf16, BH, T, first, n, D, f_lo, f_hi, gscale, codes, scales, cap, t0, scale_layout, p))
    return rc;
  if (p.nblocks == 0) return NVFP4_OK;
  cudaStream_t s = S(stream);
  const int rc = rotate ? launch_quantize_t<SRC_KV, true>(DT_BF16, p, s) : launch_quantize_t<SRC_KV, false>(DT_BF16, p, s);
  if (rc) return rc;
  return check_finite_sync(gscale, s);
}

int nvfp4_kv_append_batch(const nvfp4_kv_append_desc* descs, int count, int f_lo, int f_hi, void* stream) {
  if (count < 0 || count > NVFP4_KV_APPEND_BATCH_MAX || (count > 0 && descs == nullptr)) return NVFP4_ERR_ARG;
  if (!window_ok(f_lo, f_hi) || f_hi - f_lo + 1 > 32) return NVFP4_ERR_ARG;
  static_assert(NVFP4_KV_APPEND_BATCH_MAX == kKvBatchMax, "batch bound");
  KvBatchParams bp{};
  int m = 0;
  int64_t total = 0;
  for (int k = 0; k < count; ++k) {
    const nvfp4_kv_append_desc& d = descs[k];
    QuantParams p{};
    if (d.rotate != 0 && d.rotate != 1) return NVFP4_ERR_ARG;
    if (int rc = kv_append_params(d.k_bf16, d.BH, d.T, d.first, d.n, d.D, f_lo, f_hi, d.gscale, d.codes, d.scales,
                                  d.cap, d.t0, d.scale_layout, p))
      return rc;
    if (p.nblocks == 0) continue;
    bp.q[m] = p;
    bp.rot[m] = d.rotate;
    bp.start[m] = total;
    total += p.nblocks;   // each item < 2^32 blocks, at most 64 items
    ++m;
  }
  if (m == 0) return NVFP4_OK;
  bp.count = m;
  bp.start[m] = total;
  const int nc = f_hi - f_lo + 1;
  const bool one_per_lane = total * (nc <= 16 ? 16 : 32) <= g_lane1_max.load(std::memory_order_relaxed);
  const int64_t lanes = one_per_lane ? (nc <= 16 ? 16 : 32) : (nc <= 12 ? 4 : 8);
  // every item is below 2^32 blocks, but 64 of them can ask for more CTAs than a grid holds
  const int64_t ctas = (total * lanes + 255) / 256;
  if (ctas > INT_MAX) return NVFP4_ERR_SIZE;
  const int grid = (int)ctas;
  cudaStream_t s = S(stream);
  if (one_per_lane) {
    if (nc <= 16) kv_append_batch_kernel<16, 1><<<grid, 256, 0, s>>>(bp);
    else kv_append_batch_kernel<32, 1><<<grid, 256, 0, s>>>(bp);
  } else {
    if (nc <= 12) kv_append_batch_kernel<4, 3><<<grid, 256, 0, s>>>(bp);
    else kv_append_batch_kernel<8, 4><<<grid, 256, 0, s>>>(bp);
  }
  if (int rc = last_error()) return rc;
  for (int k = 0; k < m; ++k) {
    if (int rc = check_finite_sync(bp.q[k].g_src, s)) return rc;
  }
  return NVFP4_OK;
}

int nvfp4_kv_mixed(const void* k_bf16, int64_t B, int64_t H, int64_t T, int64_t D, int sink_tokens,
                   int recent_tokens, int rotate, int f_lo, int f_hi, void* sink_bf16, void* recent_bf16,
                   uint8_t* codes, uint8_t* scales, float* gscale, void* stream) {
  return kv_mixed_impl(k_bf16, B, H, T, D, sink_tokens, recent_tokens, rotate, f_lo, f_hi, sink_bf16, recent_bf16,
                       codes, scales, gscale, false, stream);
}

int nvfp4_kv_mixed_dequantize(const void* k_bf16, int64_t B, int64_t H, int64_t T, int64_t D, int sink_tokens,
                              int recent_tokens, int rotate, int f_lo, int f_hi, void* sink_bf16, void* recent_bf16,
                              uint8_t* codes, uint8_t* scales, float* gscale, void* mid_out, void* stream) {
  if (B > 0 && H > 0 && T > (int64_t)sink_tokens + recent_tokens && mid_out == nullptr) return NVFP4_ERR_ARG;
  return kv_mixed_impl(k_bf16, B, H, T, D, sink_tokens, recent_tokens, rotate, f_lo, f_hi, sink_bf16, recent_bf16,
                       codes, scales, gscale, false, stream, mid_out);
}

int nvfp4_kv_mixed_mma(const void* k_bf16, int64_t B, int64_t H, int64_t T, int64_t D, int sink_tokens,
                       int recent_tokens, int rotate, int f_lo, int f_hi, void* sink_bf16, void* recent_bf16,
                       uint8_t* codes, uint8_t* sf, float* gscale, void* stream) {
  return kv_mixed_impl(k_bf16, B, H, T, D, sink_tokens, recent_tokens, rotate, f_lo, f_hi, sink_bf16, recent_bf16,
                       codes, sf, gscale, true, stream);
}

}  // extern "C"
