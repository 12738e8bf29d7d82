// Host helpers of the tcgen05 kernels: TMA tensor-map encoding.
#include <cudaTypedefs.h>

#include <atomic>

#include "tc_host.h"

namespace gdn {
namespace tc {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<void *> fn{nullptr};
  void *f = fn.load(std::memory_order_acquire);
  if (!f) {
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn.store(f, std::memory_order_release);
  }
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

// bf16 tensor [BH, F, L, d] as a 4-D map with 128-byte swizzled boxes of 64 x rows.
bool make_bf16_map(CUtensorMap *m, const void *base, int d, int L, int F, int BH, int rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)F, (cuuint64_t)BH};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)L * d * 2, (cuuint64_t)F * L * d * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace gdn
