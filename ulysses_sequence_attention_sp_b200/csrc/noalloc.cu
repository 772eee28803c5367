// Allocation-free variant of the Ulysses block.
//
// usp_ulysses_attention needs a scratch workspace (the head-sharded q, k and v
// of all ranks) that its caller allocates. Some callers cannot allocate device
// memory at the point of the call: a plugin or custom operator whose host
// framework owns all device memory and hands it only the inputs and outputs,
// or code on a path that must not synchronise the device (cudaFree does). For
// them, usp_ulysses_attention_noalloc takes its scratch from a fixed array in
// this library's device memory instead.
//
// The array is a file-scope __device__ variable of kScratchBytes. Every GPU
// that loads the library holds it until the process exits. All calls share
// it: two calls that overlap on the GPU (different streams, or different
// host threads) race on it, so callers must order them. The array keeps
// the last call's contents; nothing in it needs to start at zero, because
// every call writes each element it later reads (the seq->head exchange
// fills the q, k and v head shards before the attention reads them).
#include "usp_internal.h"

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(USP_NOALLOC_SCRATCH_BYTES);

static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

}  // namespace

// In host code the array's name is only a host-side stand-in, never a device
// address: the address is looked up on the current device, once per plan, when
// the plan is created (usp_plan_create*), and kept in the plan, which lives no
// longer than the CUDA context it was made in. The lookup loads this file's
// module if it is not loaded yet, which is when the array is reserved.
int usp::noalloc_scratch_lookup(void** out) {
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess) return usp::cuda_check(e, "cudaGetSymbolAddress(allocation-free scratch)");
  *out = ptr;
  return USP_OK;
}

extern "C" int usp_ulysses_attention_noalloc(const usp_plan* plan, const void* const* q, const void* const* k,
                                             const void* const* v, void* const* out, float scale,
                                             int32_t num_chunks, void* stream) {
  if (!plan) return usp::set_error(USP_ERR_INVALID_ARG, "plan is NULL");
  size_t need = 0;
  if (int rc = usp_ulysses_attention_workspace_size(plan, num_chunks, &need)) return rc;
  if (need > kScratchBytes)
    return usp::set_error(USP_ERR_SHAPE,
                          "usp_ulysses_attention_noalloc: this plan needs %zu bytes of scratch, above the fixed "
                          "%zu-byte array; use usp_ulysses_attention with a caller-owned workspace",
                          need, kScratchBytes);
  if (!plan->noalloc_scratch) return usp::set_error(USP_ERR_INVALID_ARG, "plan has no scratch address");
  return usp_ulysses_attention(plan, q, k, v, out, scale, num_chunks, plan->noalloc_scratch, kScratchBytes,
                               stream);
}
