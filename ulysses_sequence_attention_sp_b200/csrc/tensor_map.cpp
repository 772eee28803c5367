// Host-side TMA tensor maps for the attention kernels' 4-D operand views.
#include <mutex>

#include "usp_internal.h"

namespace usp {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

}  // namespace

int make_map(CUtensorMap* map, const void* base, const AttnView& view, const AttnLaunch& L, int64_t rows, int atom,
             int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return set_error(USP_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int e = 2;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(L.head_dim), static_cast<cuuint64_t>(view.head_extent),
                        static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(L.batch)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(view.stride_head * e), static_cast<cuuint64_t>(view.stride_token * e),
                           static_cast<cuuint64_t>(view.stride_batch * e)};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(atom), 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUtensorMapSwizzle swz = atom == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                      : (atom == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  CUtensorMapDataType dt = L.dtype == USP_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(USP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return USP_OK;
}


}  // namespace usp
