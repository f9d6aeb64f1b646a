// gemm_nvfp4.cu -- NVFP4 x NVFP4 product on the sm_100a tensor cores (block-scaled tcgen05.mma, FP32
// accumulation in TMEM), consuming the quantizer's packed E2M1 codes and its E4M3 scales in the
// tensor-core tile layout directly.
//
// "Search your block floating-point scales!" (gist.science summary of arXiv 2605.12464), Method >
// ScaleSearchAttention: QK^T and PV run as NVFP4 products on the tensor cores with FP32 accumulation,
// so the ScaleSearch output is consumed without a dequantize pass.  This file provides that consumer as
// a batched A B^T product, D[l] = alpha * g_a * g_b * A[l] B[l]^T, with A [M, K] and B [N, K] both
// quantized along K (16-element blocks), which is the shape of Q K^T with K = head_dim and of a
// linear layer with activations and weights quantized along the input features.
//
// The mainloop is CUTLASS's sm100 block-scaled collective (TMA tiles into shared memory, one elected
// thread issuing the MMAs, scale factors staged through TMEM), instantiated here with a 128x128x256
// tile on one SM (a 1x1x1 cluster: every tile is loaded by the CTA that uses it).
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "cutlass/cutlass.h"
#include "cute/tensor.hpp"
#include "cutlass/detail/sm100_blockscaled_layout.hpp"
#include "cutlass/epilogue/collective/collective_builder.hpp"
#include "cutlass/gemm/collective/collective_builder.hpp"
#include "cutlass/gemm/device/gemm_universal_adapter.h"
#include "cutlass/gemm/kernel/gemm_universal.hpp"
#include "cutlass/util/packed_stride.hpp"

#include "../../include/nvfp4.h"

namespace nvfp4_consumer {

using namespace cute;

using ElementAB = cutlass::nv_float4_t<cutlass::float_e2m1_t>;
using Acc = float;
using MmaTile = Shape<_128, _128, _256>;
using ClusterShape = Shape<_1, _1, _1>;

template <class ElementD>
struct Nvfp4Gemm {
  static constexpr int kAlignD = 128 / cutlass::sizeof_bits<ElementD>::value;
  using Epilogue = typename cutlass::epilogue::collective::CollectiveBuilder<
      cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, MmaTile, ClusterShape,
      cutlass::epilogue::collective::EpilogueTileAuto, Acc, Acc, void, cutlass::layout::RowMajor, kAlignD, ElementD,
      cutlass::layout::RowMajor, kAlignD, cutlass::epilogue::collective::EpilogueScheduleAuto>::CollectiveOp;
  using Mainloop = typename cutlass::gemm::collective::CollectiveBuilder<
      cutlass::arch::Sm100, cutlass::arch::OpClassBlockScaledTensorOp, ElementAB, cutlass::layout::RowMajor, 32,
      ElementAB, cutlass::layout::ColumnMajor, 32, Acc, MmaTile, ClusterShape,
      cutlass::gemm::collective::StageCountAutoCarveout<static_cast<int>(sizeof(typename Epilogue::SharedStorage))>,
      cutlass::gemm::collective::KernelScheduleAuto>::CollectiveOp;
  using Kernel = cutlass::gemm::kernel::GemmUniversal<Shape<int, int, int, int>, Mainloop, Epilogue, void>;
  using Gemm = cutlass::gemm::device::GemmUniversalAdapter<Kernel>;
  using SfConfig = typename Mainloop::Sm1xxBlkScaledConfig;

  static int run(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb, int batch, int M,
                 int N, int K, const float* alpha_dev, void* d, cudaStream_t s) {
    auto sA = cutlass::make_cute_packed_stride(typename Mainloop::StrideA{}, make_shape(M, K, batch));
    auto sB = cutlass::make_cute_packed_stride(typename Mainloop::StrideB{}, make_shape(N, K, batch));
    auto sD = cutlass::make_cute_packed_stride(typename Epilogue::StrideD{}, make_shape(M, N, batch));
    auto lA = SfConfig::tile_atom_to_shape_SFA(make_shape(M, N, K, batch));
    auto lB = SfConfig::tile_atom_to_shape_SFB(make_shape(M, N, K, batch));
    typename Gemm::Arguments args{
        cutlass::gemm::GemmUniversalMode::kGemm,
        {M, N, K, batch},
        {reinterpret_cast<typename Mainloop::ArrayElementA const*>(a), sA,
         reinterpret_cast<typename Mainloop::ArrayElementB const*>(b), sB,
         reinterpret_cast<typename Mainloop::ElementSF const*>(sfa), lA,
         reinterpret_cast<typename Mainloop::ElementSF const*>(sfb), lB},
        {{}, nullptr, typename Epilogue::StrideC{}, static_cast<ElementD*>(d), sD}};
    args.epilogue.thread.alpha_ptr = alpha_dev;
    args.epilogue.thread.beta = 0.0f;
    Gemm gemm;
    if (Gemm::get_workspace_size(args) != 0) return NVFP4_ERR_ARG;  // this configuration needs none
    if (gemm.can_implement(args) != cutlass::Status::kSuccess) return NVFP4_ERR_SIZE;
    if (gemm.initialize(args, nullptr, s) != cutlass::Status::kSuccess) return NVFP4_ERR_CUDA;
    if (gemm.run(s) != cutlass::Status::kSuccess) return NVFP4_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
  }

  // Byte offsets the consumer reads for scale (l, r, c) of a batch of [rows, K] operands (host only).
  static void offsets(int64_t rows, int64_t K, int64_t batch, int64_t* out) {
    auto l = SfConfig::tile_atom_to_shape_SFA(make_shape((int)rows, 1, (int)K, (int)batch));
    int64_t i = 0;
    for (int64_t b = 0; b < batch; ++b)
      for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < K / 16; ++c) out[i++] = (int64_t)l((int)r, (int)(16 * c), (int)b);
  }
};

// alpha * g_a * g_b for the epilogue (one FP32 rounding after each multiply).
__global__ void gemm_alpha_kernel(const float* ga, const float* gb, float alpha, float* out) {
  if (threadIdx.x == 0 && blockIdx.x == 0) *out = __fmul_rn(__fmul_rn(alpha, *ga), *gb);
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The epilogue's scale word for nvfp4_gemm_nt_noalloc, in memory the library itself carries: a
// file-scope device array, created on every GPU that loads the library and kept until the process exits.
// It holds one FP32 word (padded to 256 bytes); the product needs that word whatever its sizes.
constexpr int kAlphaScratchFloats = 1;
static __device__ __align__(256) float g_alpha_scratch[kAlphaScratchFloats];

// Device address of g_alpha_scratch on the current device, looked up once per device (host code sees only
// a host-side stand-in under that name, so the address has to come from the runtime).
constexpr int kMaxDevices = 64;
int alpha_scratch_address(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
  static std::mutex mu;
  static float* addr[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_alpha_scratch) != cudaSuccess || p == nullptr) return NVFP4_ERR_CUDA;
    addr[dev] = static_cast<float*>(p);
  }
  *out = addr[dev];
  return NVFP4_OK;
}

}  // namespace nvfp4_consumer

using namespace nvfp4_consumer;

extern "C" {

int nvfp4_gemm_nt(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gscale, const uint8_t* b_codes,
                  const uint8_t* b_sf, const float* b_gscale, int64_t batch, int64_t M, int64_t N, int64_t K,
                  float alpha, void* d, int d_dtype, float* alpha_work, void* stream) {
  if (d_dtype != NVFP4_F32 && d_dtype != NVFP4_BF16) return NVFP4_ERR_ARG;
  if (batch < 0 || M < 0 || N < 0 || K < 0) return NVFP4_ERR_ARG;
  const int64_t lim = (int64_t(1) << 31) - 1;
  if (K % 32 != 0 || batch > lim || M > lim || N > lim || K > lim) return NVFP4_ERR_SIZE;
  int64_t t;   // every buffer's element count must fit in int64 (no wrapped size passes a later check)
  if (__builtin_mul_overflow(batch, M, &t) || __builtin_mul_overflow(t, N, &t) || __builtin_mul_overflow(t, 4, &t) ||
      __builtin_mul_overflow(batch, M, &t) || __builtin_mul_overflow(t, K, &t) ||
      __builtin_mul_overflow(batch, N, &t) || __builtin_mul_overflow(t, K, &t))
    return NVFP4_ERR_SIZE;
  if (batch == 0 || M == 0 || N == 0) return NVFP4_OK;
  if (d == nullptr) return NVFP4_ERR_ARG;
  const int esize = d_dtype == NVFP4_F32 ? 4 : 2;
  if (!aligned(d, 16) || (N * esize) % 16 != 0) return NVFP4_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) {
    return cudaMemsetAsync(d, 0, (size_t)(batch * M * N * esize), s) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
  }
  if (!a_codes || !a_sf || !a_gscale || !b_codes || !b_sf || !b_gscale || !alpha_work) return NVFP4_ERR_ARG;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_sf, 16) || !aligned(b_sf, 16) ||
      !aligned(a_gscale, 4) || !aligned(b_gscale, 4) || !aligned(alpha_work, 4))
    return NVFP4_ERR_ALIGN;
  gemm_alpha_kernel<<<1, 32, 0, s>>>(a_gscale, b_gscale, alpha, alpha_work);
  if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
  if (d_dtype == NVFP4_F32)
    return Nvfp4Gemm<float>::run(a_codes, a_sf, b_codes, b_sf, (int)batch, (int)M, (int)N, (int)K, alpha_work, d, s);
  return Nvfp4Gemm<cutlass::bfloat16_t>::run(a_codes, a_sf, b_codes, b_sf, (int)batch, (int)M, (int)N, (int)K,
                                             alpha_work, d, s);
}

int nvfp4_gemm_nt_noalloc(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gscale,
                          const uint8_t* b_codes, const uint8_t* b_sf, const float* b_gscale, int64_t batch,
                          int64_t M, int64_t N, int64_t K, float alpha, void* d, int d_dtype, void* stream) {
  float* work = nullptr;
  if (int rc = alpha_scratch_address(&work)) return rc;
  return nvfp4_gemm_nt(a_codes, a_sf, a_gscale, b_codes, b_sf, b_gscale, batch, M, N, K, alpha, d, d_dtype, work,
                       stream);
}

int nvfp4_gemm_sf_offsets(int64_t rows, int64_t K, int64_t batch, int64_t* out) {
  if (rows <= 0 || K <= 0 || batch <= 0 || K % 16 != 0 || out == nullptr) return NVFP4_ERR_ARG;
  if (rows > (int64_t(1) << 30) || K > (int64_t(1) << 30) || batch > (int64_t(1) << 20)) return NVFP4_ERR_SIZE;
  Nvfp4Gemm<float>::offsets(rows, K, batch, out);
  return NVFP4_OK;
}

}  // extern "C"
