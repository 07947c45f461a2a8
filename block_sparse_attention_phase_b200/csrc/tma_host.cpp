// Host-side TMA tensor-map encoding. The driver's cuTensorMapEncodeTiled is
// looked up through the runtime (cudaGetDriverEntryPoint), so the library does
// not link libcuda directly and loads on machines without a GPU driver.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "star_internal.h"

namespace star {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      return nullptr;
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

}  // namespace

bool encode_tma_bf16_4d(void* tmap_out, const void* base, uint64_t d, uint64_t heads,
                        uint64_t tokens, uint64_t token_rows, uint64_t batch, uint32_t box0,
                        uint32_t box1, uint32_t box2, bool swizzle128) {
  if (tokens > token_rows) return false;
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {d, heads, tokens, batch};
  const cuuint64_t strides[3] = {d * 2, heads * d * 2, token_rows * heads * d * 2};
  const cuuint32_t box[4] = {box0, box1, box2, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(static_cast<CUtensorMap*>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace star
