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
#include <mutex>

#include "usp_internal.h"

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(USP_NOALLOC_SCRATCH_BYTES);

static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device. In host
// code the array's name is only a host-side stand-in, never a device address.
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

int scratch_address(int device, void** out) {
  if (device < 0 || device >= kMaxDevices)
    return usp::set_error(USP_ERR_UNSUPPORTED, "device ordinal %d is beyond %d", device, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[device]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return usp::cuda_check(e, "cudaGetSymbolAddress(scratch)");
    g_scratch_ptr[device] = ptr;
  }
  *out = g_scratch_ptr[device];
  return USP_OK;
}

}  // namespace

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
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return usp::cuda_check(e, "cudaGetDevice");
  void* scratch = nullptr;
  if (int rc = scratch_address(device, &scratch)) return rc;
  return usp_ulysses_attention(plan, q, k, v, out, scale, num_chunks, scratch, kScratchBytes, stream);
}
