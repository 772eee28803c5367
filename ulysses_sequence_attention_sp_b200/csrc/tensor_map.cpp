// Host-side TMA tensor maps: the attention kernels' 4-D operand views and the
// TMA pack's row tiles, encoded through the driver's cuTensorMapEncodeTiled.
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

int encode_tiled_4d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t dims[4],
                    const uint64_t strides_bytes[3], const uint32_t box[4], CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return set_error(USP_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t st[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
  cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, dtype, 4, const_cast<void*>(base), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(USP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return USP_OK;
}

int make_map(CUtensorMap* map, const void* base, const AttnView& view, const AttnLaunch& L, int64_t rows, int atom,
             int box_rows) {
  const int e = 2;
  const uint64_t dims[4] = {static_cast<uint64_t>(L.head_dim), static_cast<uint64_t>(view.head_extent),
                            static_cast<uint64_t>(rows), static_cast<uint64_t>(L.batch)};
  const uint64_t strides[3] = {static_cast<uint64_t>(view.stride_head * e), static_cast<uint64_t>(view.stride_token * e),
                               static_cast<uint64_t>(view.stride_batch * e)};
  const uint32_t box[4] = {static_cast<uint32_t>(atom), 1, static_cast<uint32_t>(box_rows), 1};
  const CUtensorMapSwizzle swz = atom == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                            : (atom == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  const CUtensorMapDataType dt =
      L.dtype == USP_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return encode_tiled_4d(map, dt, base, dims, strides, box, swz);
}

}  // namespace usp
